/*
 * plx.h -- C ABI of libplx.so: the Parallax attention forward pass on
 * NVIDIA B200 (sm_100a).
 *
 * The operation.  For each query i (per batch entry b and query head h):
 *
 *     w_ij   = softmax_j(scale * q_i . k_j)            over the key set J_i
 *     o_SA_i = sum_j w_ij v_j
 *     Sigma_i = sum_j w_ij (v_j - o_SA_i)(k_j - k_bar_i)^T,  k_bar_i = sum_j w_ij k_j
 *     out_i  = o_SA_i - Sigma_i rho_i
 *     lse_i  = ln sum_j exp(scale * q_i . k_j)
 *
 * This is the output equation of gist.science, "Technical overview:
 * Parallax - parameterized local linear attention for language modeling",
 * section "Method: Parallax / Core mechanism", with the boundary
 * amplification factor eta set to zero as the same section states; the
 * softmax-weighted, un-Bessel-corrected covariance and the unscaled probe
 * score s_ij = rho_i . k_j are the plain readings of that equation.  The
 * kernels compute it in the streamed form of news.chathome.org, "Parallax:
 * a parameterized local linear attention ...", section "Hardware argument":
 * two score branches (q.k and rho.k) that share one online max, one
 * rescale factor and the same K/V tiles, accumulating l = sum p,
 * c = sum p s, O1 = sum p v and O2 = sum p s v and emitting
 * out = O1/l - (O2/l - (c/l)(O1/l)).
 *
 * Conventions shared by every entry point
 *   - Tensors are dense, row-major, bf16 (IEEE bfloat16 stored as uint16)
 *     unless stated; every pointer is a DEVICE pointer, 16-byte aligned.
 *   - GQA: query head h reads key/value head h / (Hq / Hkv); Hq % Hkv == 0.
 *     rho (argument r) is given per query head.
 *   - Head dimension d (= d_k = d_v) is 64 or 128.
 *   - scale multiplies q.k only; pass 1/sqrt(d) for the usual choice.
 *   - r == NULL means rho = 0, which is exactly softmax attention (the same
 *     page, section "How the mechanism works": probe norm zero reduces to
 *     softmax); the kernels then skip the rho branch.
 *   - lse may be NULL (not written).
 *   - The caller owns every buffer.  The library allocates no device or
 *     host memory; it keeps one device word that records a bounded-wait
 *     timeout (see plx_check_device_status) and one fixed scratch array for
 *     plx_decode_noalloc.
 *   - stream is a cudaStream_t (NULL = legacy default stream).  Calls are
 *     asynchronous on it.  Argument errors are returned synchronously
 *     before anything is launched; launch failures return PLX_ERR_CUDA.
 *   - Return value: a plx_status (0 = PLX_OK, negative = error).
 */
#ifndef PLX_H_
#define PLX_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum plx_status {
  PLX_OK = 0,
  PLX_ERR_NULL = -1,            /* a required pointer is NULL */
  PLX_ERR_SHAPE = -2,           /* a size is out of range (B, H, N, S_max < 1, ...) */
  PLX_ERR_HEADDIM = -3,         /* d not in {64, 128} */
  PLX_ERR_GQA = -4,             /* Hq % Hkv != 0 */
  PLX_ERR_ALIGN = -5,           /* a pointer is not 16-byte aligned */
  PLX_ERR_WORKSPACE = -6,       /* workspace NULL or smaller than required */
  PLX_ERR_CUDA = -7,            /* a CUDA runtime/driver call failed */
  PLX_ERR_DEVICE_TIMEOUT = -8,  /* a kernel gave up a bounded wait (device word set) */
  PLX_ERR_ARCH = -9             /* current device is not sm_100 */
} plx_status;

/* Library version, major*10000 + minor*100 + patch. */
int plx_version(void);

/* Human-readable name of a status code (static string, never NULL). */
const char* plx_status_string(int status);

/*
 * plx_fwd -- prefill / full-sequence forward.
 *
 *   q   [B, Hq,  N, d] bf16   queries
 *   k   [B, Hkv, N, d] bf16   keys
 *   v   [B, Hkv, N, d] bf16   values
 *   r   [B, Hq,  N, d] bf16   probes rho (NULL: rho = 0)
 *   out [B, Hq,  N, d] bf16   output (written)
 *   lse [B, Hq,  N]    fp32   natural-log LSE of the scaled q.k scores (NULL: skipped)
 *   causal != 0: J_i = {j <= i} (diagonal included); causal == 0: all j < N.
 *
 * Requirements: B, Hq, Hkv, N >= 1; d in {64, 128}; Hq % Hkv == 0;
 * all pointers 16-byte aligned; out must not alias an input.
 * Runs one kernel (tcgen05 tensor cores, TMA-fed) on `stream`.
 */
int plx_fwd(const void* q, const void* k, const void* v, const void* r,
            void* out, float* lse,
            int B, int Hq, int Hkv, int N, int d, int causal, float scale,
            void* stream);

/*
 * plx_fwd_varlen -- plx_fwd over a batch of packed sequences of different
 * lengths (variable-length prefill).
 *
 *   q, r, out [total, Hq, d] bf16; k, v [total, Hkv, d] bf16   token-major:
 *              sequence b is tokens cu_seqlens[b] .. cu_seqlens[b+1]-1
 *   cu_seqlens [B + 1] int32, DEVICE   non-decreasing, cu_seqlens[0] = 0,
 *              cu_seqlens[B] = total
 *   lse [Hq, total] fp32 (NULL: skipped)
 *   max_seqlen >= every sequence's length (rows past it are not computed)
 *
 * Each sequence attends only its own tokens (causal: positions within the
 * sequence).  Values in cu_seqlens outside [0, total] are clamped on the
 * device, so nothing outside the tensors is addressed.  Same requirements
 * and errors as plx_fwd, plus PLX_ERR_NULL for cu_seqlens and PLX_ERR_SHAPE
 * for total < 1.  The pages train on fixed-length windows; packing is the
 * serving / mixed-length form of the same computation.
 */
int plx_fwd_varlen(const void* q, const void* k, const void* v, const void* r,
                   void* out, float* lse, const int32_t* cu_seqlens,
                   int B, int Hq, int Hkv, int total, int max_seqlen, int d, int causal,
                   float scale, void* stream);

/*
 * Context-parallel prefill.  The sequence is cut into consecutive chunks, one
 * per rank.  A rank's queries attend its own chunk causally and every earlier
 * chunk in full; each (query chunk, key chunk) block yields one partial state
 * per query row, and the merge combines them.  The partial state over a set
 * of keys is the streamed form's 5-tuple (news.chathome.org, "Parallax: ...",
 * section "Hardware argument"): m (running max of the scaled scores, log2
 * units), l = sum p, c = sum p s, O1 = sum p v, O2 = sum p s v.  Rescaled to a
 * common max, the tuples of disjoint key sets add, so the merged output is
 * o = O1/l - (O2/l - (c/l)(O1/l)) over the union of the keys.
 *
 * plx_fwd_partial_size -- bytes of one block: B * Hq * N * (2d + 4) fp32
 *   (0 for invalid shapes).
 */
size_t plx_fwd_partial_size(int B, int Hq, int N, int d);

/*
 * plx_fwd_partial -- the partial states of the queries q against the keys
 * k, v (one block).
 *   q, r [B, Hq, N, d] bf16; k, v [B, Hkv, N, d] bf16: as plx_fwd, where the
 *     N keys are one chunk (the query chunk itself with causal != 0, an
 *     earlier chunk with causal == 0).
 *   partial [B, Hq, N, 2d + 4] fp32, DEVICE, written: per query row m (log2
 *     units; -inf for a row that saw no key), l, c, pad, O1[d], O2[d], with
 *     l, c, O1, O2 relative to 2^m.
 * Requirements and errors as plx_fwd; PLX_ERR_NULL for partial,
 * PLX_ERR_WORKSPACE when partial_bytes < plx_fwd_partial_size.  One kernel
 * (the prefill kernel with a partial-state epilogue) on `stream`.
 */
int plx_fwd_partial(const void* q, const void* k, const void* v, const void* r,
                    float* partial, size_t partial_bytes,
                    int B, int Hq, int Hkv, int N, int d, int causal, float scale,
                    void* stream);

/*
 * plx_fwd_merge -- out and lse from `ranks` blocks of partial states.
 *   partials [ranks, B, Hq, N, 2d + 4] fp32, DEVICE (block-major)
 *   out [B, Hq, N, d] bf16; lse [B, Hq, N] fp32 (NULL: skipped)
 * A row with no live key in any block gives out = 0, lse = -inf.  Errors:
 * PLX_ERR_NULL, PLX_ERR_SHAPE (ranks, B, Hq or N < 1), PLX_ERR_HEADDIM,
 * PLX_ERR_ALIGN (partials and out 16-byte, lse 4-byte aligned).
 */
int plx_fwd_merge(const float* partials, int ranks, int B, int Hq, int N, int d,
                  void* out, float* lse, void* stream);

/*
 * plx_fwd_train -- plx_fwd for training: the same outputs, plus two per-row
 * values that plx_bwd needs.
 *
 *   obar [B, Hq, N, d] bf16   o_bar_i = sum_j w_ij v_j, the softmax-attention
 *                             output inside the Parallax output equation
 *   sbar [B, Hq, N]    fp32   s_bar_i = sum_j w_ij (rho_i . k_j); may be NULL
 *                             only when r is NULL (then s_bar = 0)
 *   lse must not be NULL here.
 *
 * Both are exact by-products of the streamed form (O1 / l and c / l).  The
 * pages give the forward only; keeping them is this library's choice, so that
 * the backward needs no extra pass over the keys.  Returns PLX_ERR_NULL when
 * lse or obar is NULL, or sbar is NULL with r non-NULL; otherwise as plx_fwd.
 */
int plx_fwd_train(const void* q, const void* k, const void* v, const void* r,
                  void* out, float* lse, void* obar, float* sbar,
                  int B, int Hq, int Hkv, int N, int d, int causal, float scale,
                  void* stream);

/*
 * plx_bwd_workspace_size -- bytes of device workspace plx_bwd needs: two fp32
 * values per query row (g_bar and Dd below), each array padded to 256 bytes.
 * 0 for invalid sizes.
 */
size_t plx_bwd_workspace_size(int B, int Hq, int Hkv, int N, int d);

/*
 * plx_bwd -- gradients of the loss sum_i dout_i . out_i with respect to q, k,
 * v and rho, for the forward of plx_fwd_train with the same arguments.
 *
 * The pages define the forward only (gist.science, section "Method: Parallax
 * / Core mechanism").  Written with effective weights
 * w_hat_ij = w_ij (1 - s_ij + s_bar_i), s_ij = rho_i . k_j, its gradient is
 *   g_ij = dout_i . v_j, g_bar_i = dout_i . obar_i, Dd_i = dout_i . out_i + s_bar_i g_bar_i
 *   dv_j = sum_i w_hat_ij dout_i
 *   dS_ij = w_ij (g_bar_i - g_ij),  dA_ij = w_ij (g_ij (1 - s_ij + s_bar_i) + s_ij g_bar_i - Dd_i)
 *   dq_i = scale sum_j dA_ij k_j,  dr_i = sum_j dS_ij k_j,
 *   dk_j = sum_i scale dA_ij q_i + dS_ij rho_i
 * with w_ij = exp(scale q_i . k_j - lse_i).
 *
 *   q, r [B, Hq, N, d] bf16; k, v [B, Hkv, N, d] bf16   forward inputs (r NULL: rho = 0)
 *   out, obar [B, Hq, N, d] bf16; lse, sbar [B, Hq, N] fp32   from plx_fwd_train
 *                                                    (sbar ignored when r is NULL)
 *   dout [B, Hq, N, d] bf16                          gradient of the loss w.r.t. out
 *   dq, dr [B, Hq, N, d] bf16; dk, dv [B, Hkv, N, d] bf16   written (dr may be NULL;
 *                                                    with r NULL it is the gradient at rho = 0)
 *   workspace: at least plx_bwd_workspace_size(...) bytes, 16-byte aligned;
 *   its contents are overwritten.
 *
 * Runs three kernels on `stream`: a per-row reduction, a query-side kernel
 * (dq, dr) and a key-side kernel (dk, dv), both on tcgen05 tensor cores.  The
 * outputs are written, not accumulated; dk and dv sum over the query heads
 * of each KV group.  Requirements and errors as plx_fwd, plus
 * PLX_ERR_WORKSPACE for a missing or small workspace.
 */
int plx_bwd(const void* q, const void* k, const void* v, const void* r,
            const void* out, const void* dout, const float* lse,
            const void* obar, const float* sbar,
            void* dq, void* dk, void* dv, void* dr,
            int B, int Hq, int Hkv, int N, int d, int causal, float scale,
            void* workspace, size_t workspace_bytes, void* stream);

/*
 * plx_decode_num_splits -- the split count plx_decode uses when passed
 * num_splits = 0 (a function of the shapes only; >= 1).
 */
int plx_decode_num_splits(int B, int Hq, int Hkv, int S_max, int d);

/*
 * plx_decode_workspace_size -- bytes of workspace plx_decode needs for these
 * shapes and split count (0 = the automatic count).  0 when one split is used.
 */
size_t plx_decode_workspace_size(int B, int Hq, int Hkv, int S_max, int d, int num_splits);

/*
 * plx_decode -- one decode step against a KV cache, split over the keys.
 *
 *   q       [B, Hq, d]           bf16   one query per (b, h)
 *   r       [B, Hq, d]           bf16   its probe rho (NULL: rho = 0)
 *   kcache  [B, Hkv, S_max, d]   bf16   key cache
 *   vcache  [B, Hkv, S_max, d]   bf16   value cache
 *   seqlens [B]                  int32  DEVICE array; query (b, .) attends the
 *                                       cached keys j < seqlens[b] (values above
 *                                       S_max are clamped to S_max; <= 0 gives
 *                                       out = 0 and lse = -inf)
 *   out     [B, Hq, d]           bf16   output (written)
 *   lse     [B, Hq]              fp32   (NULL: skipped)
 *   num_splits: 0 = automatic.  A positive count asks for the balanced plan
 *     with that many persistent CTAs, which take equal ranges of the batch's
 *     64-key tiles; a (b, kv head) stream cut by a range boundary leaves a
 *     partial state (m, l, c, O1, O2) per CTA in `workspace`, and a second
 *     kernel merges them.  The automatic choice may instead take the chunked
 *     plan (a split-KV grid and a merge kernel) for many long streams.  The
 *     result does not depend on the plan or the count beyond rounding.
 *   workspace / workspace_bytes: caller-owned device scratch of at least
 *     plx_decode_workspace_size(...) bytes, 16-byte aligned (may be NULL when
 *     that size is 0).  Its contents are overwritten; it need not start at
 *     zero.  Calls that overlap on the GPU must not share one.
 *   Cache rows at or past seqlens[b] are never used and may hold anything
 *   (NaN and Inf included).
 *
 * Requirements: B, Hq, Hkv, S_max >= 1; d in {64, 128}; Hq % Hkv == 0.
 */
int plx_decode(const void* q, const void* r, const void* kcache, const void* vcache,
               const int32_t* seqlens, void* out, float* lse,
               int B, int Hq, int Hkv, int S_max, int d, float scale, int num_splits,
               void* workspace, size_t workspace_bytes, void* stream);

/*
 * plx_decode_paged -- plx_decode against a paged KV cache (block tables).
 *
 *   kpool, vpool [num_pages, Hkv, page_size, d] bf16   page pools: page p holds
 *                page_size consecutive keys (values) of every KV head
 *   block_table  [B, max_pages] int32, DEVICE   pool page of each page slot:
 *                keys n*page_size .. (n+1)*page_size-1 of sequence b are in
 *                page block_table[b * max_pages + n]
 *   seqlens      [B] int32, DEVICE   live keys per sequence (clamped to
 *                [0, max_pages * page_size])
 *   page_size    a power of two, 16 .. 4096
 *   q, r, out, lse, scale, num_splits, workspace: as plx_decode, with
 *   S_max = max_pages * page_size (plx_decode_workspace_size and
 *   plx_decode_num_splits take that S_max).
 *
 * Reads only the table entries of pages that hold live keys.  An entry
 * outside [0, num_pages) is treated as a page of zeros (its keys then score
 * 0 and carry zero values); nothing outside the pools is read.  Keys past
 * seqlens[b] inside a live page are read and weighted 0: they must hold
 * finite values, as must the unused rows of a contiguous cache.
 * Results equal plx_decode on the gathered contiguous cache with the same
 * S_max and split count.  This is the serving form of the decode step
 * (paged caches); the pages themselves describe only a contiguous cache.
 */
int plx_decode_paged(const void* q, const void* r, const void* kpool, const void* vpool,
                     const int32_t* block_table, const int32_t* seqlens, void* out, float* lse,
                     int B, int Hq, int Hkv, int num_pages, int page_size, int max_pages,
                     int d, float scale, int num_splits,
                     void* workspace, size_t workspace_bytes, void* stream);

/*
 * plx_kv_append -- writes the new token's key and value of every KV head into
 * a contiguous cache at the slot after the live keys, before the decode step.
 *
 *   knew, vnew [B, Hkv, d] bf16          this step's keys and values
 *   kcache, vcache [B, Hkv, S_max, d]     written at row seqlens[b] of (b, g)
 *   seqlens [B] int32, DEVICE             read; when advance != 0, entry b
 *                                         becomes seqlens[b] + 1 once written
 *
 * An entry with seqlens[b] < 0 or >= S_max is left unwritten (and not
 * advanced).  One small kernel on `stream`; calls on one stream apply in
 * order.  The pages describe a KV cache that grows by one token per step
 * (zubnet.ai's Parallax page: a KV cache is still needed); this is that step.
 */
int plx_kv_append(const void* knew, const void* vnew, void* kcache, void* vcache,
                  int32_t* seqlens, int B, int Hkv, int S_max, int d, int advance, void* stream);

/*
 * plx_kv_append_paged -- plx_kv_append for the page pools of plx_decode_paged
 * ([num_pages, Hkv, page_size, d]; slot seqlens[b] of sequence b is row
 * seqlens[b] % page_size of page block_table[b * max_pages + seqlens[b] / page_size]).
 * An entry whose slot is past max_pages * page_size, or whose page id is
 * outside [0, num_pages), is left unwritten and not advanced.
 */
int plx_kv_append_paged(const void* knew, const void* vnew, void* kpool, void* vpool,
                        const int32_t* block_table, int32_t* seqlens, int B, int Hkv,
                        int num_pages, int page_size, int max_pages, int d, int advance,
                        void* stream);

/*
 * The projection in front of the attention.  The pages make the probe rho one
 * more learned projection of the layer input, beside q, k and v
 * (news.chathome.org, "Parallax: ...", section "What is Parallax"; gist.science,
 * "Technical overview: Parallax ...", "Method: Parallax / Core mechanism").  The
 * four weights are stacked along the output dimension,
 *
 *     w = [W_Q; W_K; W_V; W_R]   [Nout, d_model] bf16, row-major (a row per
 *                                output feature), Nout = (2 Hq + 2 Hkv) d,
 *                                rows: Hq*d of W_Q, Hkv*d of W_K, Hkv*d of W_V,
 *                                Hq*d of W_R (head-major, d per head);
 *                                with r == NULL the W_R rows are absent,
 *                                Nout = (Hq + 2 Hkv) d,
 *
 * and one GEMM y = x w^T (bf16 operands, fp32 accumulation, bf16 results on
 * tcgen05 tensor cores) gives all four; its epilogue writes every head's d
 * columns straight into the layout the attention reads.  No bias, no
 * normalisation, no positional rotation: the pages name none.  One kernel on
 * `stream`; no workspace.
 *
 * plx_qkvr_proj -- prefill: x [B * N, d_model] bf16 (token m = b N + t);
 *   writes q, r [B, Hq, N, d] and k, v [B, Hkv, N, d] (r may be NULL).
 * Requirements: B, N >= 1; d_model >= 8 and a multiple of 8; d in {64, 128};
 * Hq % Hkv == 0; pointers 16-byte aligned.  Errors: PLX_ERR_NULL,
 * PLX_ERR_SHAPE, PLX_ERR_HEADDIM, PLX_ERR_GQA, PLX_ERR_ALIGN, PLX_ERR_CUDA.
 */
int plx_qkvr_proj(const void* x, const void* w, void* q, void* k, void* v, void* r,
                  int B, int N, int d_model, int Hq, int Hkv, int d, void* stream);

/*
 * plx_qkvr_proj_decode -- one decode step's projection with the KV append
 * fused in: x [B, d_model] bf16 holds each sequence's new token; writes
 * q, r [B, Hq, d] and the token's k, v of every KV head into
 * kcache, vcache [B, Hkv, S_max, d] at row seqlens[b].  An entry with
 * seqlens[b] < 0 or >= S_max gets no k, v.  seqlens_out (DEVICE int32 [B],
 * may be NULL; must not be seqlens) receives seqlens[b] + 1 where the token
 * was written and seqlens[b] elsewhere: the lengths the decode step then
 * reads.  Requirements and errors as plx_qkvr_proj, plus S_max >= 1.
 */
int plx_qkvr_proj_decode(const void* x, const void* w, void* q, void* r, void* kcache, void* vcache,
                         const int32_t* seqlens, int32_t* seqlens_out, int B, int d_model, int Hq, int Hkv,
                         int S_max, int d, void* stream);

/*
 * plx_qkvr_proj_decode_paged -- plx_qkvr_proj_decode for the page pools of
 * plx_decode_paged: k, v go to row seqlens[b] % page_size of page
 * block_table[b * max_pages + seqlens[b] / page_size]; nothing is written for
 * a slot past max_pages * page_size or a page id outside [0, num_pages).
 */
int plx_qkvr_proj_decode_paged(const void* x, const void* w, void* q, void* r, void* kpool, void* vpool,
                               const int32_t* block_table, const int32_t* seqlens, int32_t* seqlens_out, int B,
                               int d_model, int Hq, int Hkv, int num_pages, int page_size, int max_pages, int d,
                               void* stream);

/*
 * Context-parallel decode: the KV cache of each sequence is split along the
 * sequence over `ranks` GPUs (rank r holds a contiguous slice of the keys).
 * Each rank computes the partial state of its slice with
 * plx_decode_partial, the ranks all-gather the partials (a collective the
 * caller runs, e.g. NCCL all-gather into [ranks, ...]), and every rank merges
 * them with plx_decode_merge.  The partial state of a set of keys is the
 * streamed form's 5-tuple (news.chathome.org, "Parallax: ...", section
 * "Hardware argument"): m (running max of the scaled scores, log2 units),
 * l = sum p, c = sum p s, O1 = sum p v, O2 = sum p s v; the merge rescales
 * each tuple to the common max and sums, as the split-KV combine does.
 *
 * plx_decode_partial_size -- bytes of the partial block of one rank:
 *   B * Hq * splits * (2d + 4) fp32, where splits is the count the kernel
 *   uses: plx_decode_num_splits for these shapes when num_splits == 0, else
 *   num_splits rounded so that every split is a whole number of 64-key tiles
 *   (the byte count gives it).  Every rank must use the same count.
 */
size_t plx_decode_partial_size(int B, int Hq, int Hkv, int S_max, int d, int num_splits);

/*
 * plx_decode_partial -- the partial states of this rank's slice of the keys.
 *   q, r, kcache, vcache, scale, num_splits: as plx_decode, where the caches
 *   hold this rank's slice [B, Hkv, S_max, d]: keys key_offset ..
 *   key_offset + S_max - 1 of every sequence.
 *   seqlens [B] int32, DEVICE: the sequences' full lengths; the slice's live
 *   keys are min(max(seqlens[b] - key_offset, 0), S_max).
 *   partial [B, Hq, splits, 2d + 4] fp32, DEVICE: per (b, h, split)
 *   m (log2 units; -inf for an empty split), l, c, pad, O1[d], O2[d].
 * Errors as plx_decode; PLX_ERR_WORKSPACE when partial_bytes is too small,
 * PLX_ERR_SHAPE for a negative key_offset.
 */
int plx_decode_partial(const void* q, const void* r, const void* kcache, const void* vcache,
                       const int32_t* seqlens, int key_offset, int B, int Hq, int Hkv, int S_max,
                       int d, float scale, int num_splits, float* partial, size_t partial_bytes,
                       void* stream);

/*
 * plx_decode_merge -- out and lse from the gathered partials of all ranks.
 *   partials [ranks, B, Hq, num_splits, 2d + 4] fp32, DEVICE (rank-major)
 *   out [B, Hq, d] bf16; lse [B, Hq] fp32 (NULL: skipped)
 * A row with no live key in any rank gives out = 0, lse = -inf.
 */
int plx_decode_merge(const float* partials, int ranks, int B, int Hq, int d,
                     void* out, float* lse, void* stream);

/*
 * PLX_NOALLOC_SCRATCH_BYTES -- size of the library's fixed device scratch
 * array used by plx_decode_noalloc (16 MiB, held on every GPU that loads the
 * library until the process exits).
 */
#define PLX_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)

/*
 * plx_decode_noalloc -- plx_decode for callers that cannot allocate device
 * memory.  Some callers have no way to call cudaMalloc, or must not: a
 * plugin inside another runtime that owns all device memory and hands the
 * plugin only its input and output buffers, or a latency-critical serving
 * loop whose host forbids device allocation after start-up (an allocation
 * can synchronise the device or fail under memory pressure).  This entry
 * point needs no workspace argument:
 * the split partial states live in a fixed device array inside the library
 * (PLX_NOALLOC_SCRATCH_BYTES).  The paper has no counterpart to this call; it
 * is a convenience of this library.
 *
 * Arguments, layouts and results are those of plx_decode (without
 * workspace / workspace_bytes); num_splits = 0 picks the automatic count.
 *   - The caller still owns and passes every input and output buffer.
 *   - Returns PLX_ERR_WORKSPACE, before launching anything, when the partial
 *     states for these shapes and this split count would need more than
 *     PLX_NOALLOC_SCRATCH_BYTES (plx_decode_workspace_size tells the need).
 *   - The first call on a device looks up that device's address of the array
 *     (cudaGetSymbolAddress, with the device current); make that first call
 *     before any stream capture.  It allocates nothing, here or later.
 *   - Every call, on every stream, shares the one array, and the array keeps
 *     the contents of the last call.  Nothing in it needs to start at zero:
 *     each call writes every partial it later reads.  Calls that overlap on
 *     the GPU (different streams without ordering between them) race on the
 *     array and give undefined results; order them, or use plx_decode with a
 *     workspace per stream.
 */
int plx_decode_noalloc(const void* q, const void* r, const void* kcache, const void* vcache,
                       const int32_t* seqlens, void* out, float* lse,
                       int B, int Hq, int Hkv, int S_max, int d, float scale, int num_splits,
                       void* stream);

/*
 * plx_check_device_status -- synchronises `stream`, then reads and clears the
 * library's device error word.  Every wait inside the kernels (on an
 * mbarrier fed by TMA or by tensor-core completion) is bounded in time; a
 * kernel that gives up sets the word, releases what it holds and returns.
 * Returns PLX_OK, PLX_ERR_DEVICE_TIMEOUT (word was set; it is now clear) or
 * PLX_ERR_CUDA.  After a timeout the outputs of calls made before this check
 * are undefined.
 */
int plx_check_device_status(void* stream);

/*
 * plx_selftest_wait_timeout -- test hook for the bounded-wait path: launches
 * one tiny kernel that waits on an mbarrier nothing ever completes, with a
 * limit of `limit_cycles` SM clock cycles, so that the wait runs out and sets
 * the device error word.  Follow with plx_check_device_status, which must
 * return PLX_ERR_DEVICE_TIMEOUT.  Faults nothing; the context stays usable.
 */
int plx_selftest_wait_timeout(unsigned long long limit_cycles, void* stream);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* PLX_H_ */
