// plx_decode.cuh -- split-KV decode for the Parallax forward pass.
//
// One CTA per (key chunk, kv head, head group, batch entry).  Every query head
// of the group reads the same key/value stream, which is read from HBM once:
// a producer warp streams 64-key K and V tiles with TMA (128-byte swizzle,
// 3-stage ring), and four consumer warps take 16 keys each per tile.
//
// Both score branches of the method -- q.k and rho.k -- come out of ONE
// tensor-core instruction: the A operand of the m16n8k16 MMA stacks the
// group's queries in rows 0..G-1 and their probes rho in rows 8..8+G-1, so a
// thread holds a_ij (row g) and s_ij (row g+8) for the same key.  (This is
// the stacking the pages describe for their decode kernel, news.chathome.org,
// "Parallax: a parameterized local linear attention ...", section "Hardware
// argument": a decode step offers one query row, so the QK and RK products
// fit inside the instruction the attention step already issues.)  The same
// stacking carries through the value product: A rows g hold p_ij and rows g+8
// hold p_ij * s_ij, giving O1 = sum p v in rows g and O2 = sum p s v in rows
// g+8 of one accumulator.  The online max and the rescale factor are shared
// by both branches (same page, same section).
//
// Each CTA writes its partial state (m, l, c, O1, O2) to the workspace, or,
// with a single split, the final out = O1/l - (O2/l - (c/l)(O1/l)) and lse.
// plx_decode_combine merges the partials of all splits.
//
// Paged caches (PAGED = true): K and V live in page pools
// [num_pages, Hkv, page_size, D] and a block table maps the page slots of
// each sequence to pool pages.  The producer looks up the page of every
// min(page_size, 64)-key part of a tile and loads it from there; a part past
// the sequence, or with a page id outside the pool, is loaded at a row past
// the page, which TMA fills with zeros, so no page outside the pool is read.
// The consumers are the same as for contiguous caches.
#pragma once

#include "plx_ptx.cuh"

namespace plx {

constexpr int kDecTileKeys = 64;     // keys per pipeline stage
constexpr int kDecConsumerWarps = 4; // 16 keys of each tile per warp
constexpr int kDecThreads = (kDecConsumerWarps + 1) * 32;

template <int D>
struct DecodeCfg {
  static constexpr int kHalves = D / 64;                       // 128-byte swizzle rows per key
  static constexpr int kTileBytes = kDecTileKeys * D * 2;      // one of K or V
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kStages = D == 128 ? 3 : 6;
  static constexpr int kSmemBytes = kStages * kStageBytes + 1024 /*align*/ + 256 /*barriers*/;
  static constexpr int kPartialFloats = 2 * D + 4;             // m, l, c, pad, O1[D], O2[D]
};

struct DecodeParams {
  const __nv_bfloat16* q;   // [B, Hq, D]
  const __nv_bfloat16* r;   // [B, Hq, D] or nullptr
  const int32_t* seqlens;   // [B]
  __nv_bfloat16* out;       // [B, Hq, D]
  const int32_t* block_table;  // [B, max_pages] pool page of each page slot (paged caches)
  int num_pages, max_pages, page_size, page_shift, box_rows;  // paged caches: pool, table width, page
  float* lse;               // [B, Hq] or nullptr
  float* ws;                // [B, Hq, splits, 2D+4] or nullptr when splits == 1
                            //   per row: m (log2 units), l, c, pad, O1[D], O2[D]
  int B, Hq, Hkv, S_max, G, n_hgroups, splits, chunk;
  int partial_out;          // 1: always write partial states to ws (context parallel), never out
  int key_offset;           // global index of the cache's first key (context parallel; else 0)
  float scale_log2;         // scale * log2(e)
};

// Byte offset of (key row, 16-byte chunk) inside one 64-key x 128-byte block
// written by TMA with CU_TENSOR_MAP_SWIZZLE_128B.
__device__ __forceinline__ uint32_t sw128(int row, int chunk) {
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

template <int D, bool HAS_R, bool PAGED>
__global__ void __launch_bounds__(kDecThreads, 2)
plx_decode_split_kernel(const __grid_constant__ CUtensorMap kmap,
                        const __grid_constant__ CUtensorMap vmap, const DecodeParams p) {
  using Cfg = DecodeCfg<D>;
  constexpr int NS = Cfg::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + NS * Cfg::kStageBytes);
  uint64_t* empty_bar = full_bar + NS;

  const int split = blockIdx.x;
  const int g = blockIdx.y / p.n_hgroups;          // kv head
  const int hg = blockIdx.y % p.n_hgroups;         // head group within the kv head
  const int b = blockIdx.z;
  const int h0 = g * p.G + hg * 8;                 // first query head of this CTA
  const int nh = min(8, p.G - hg * 8);             // live query heads (rows)
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // live keys of this cache: the sequence's keys past key_offset, at most S_max
  int seqlen = p.seqlens[b] - p.key_offset;
  seqlen = seqlen < 0 ? 0 : (seqlen > p.S_max ? p.S_max : seqlen);
  const int kbeg = split * p.chunk;
  const int kend = min(kbeg + p.chunk, seqlen);
  const int ntiles = kend > kbeg ? (kend - kbeg + kDecTileKeys - 1) / kDecTileKeys : 0;

  if (ntiles == 0) {
    // Empty chunk: an empty partial state, or (single split) the empty-set output.
    if (warp >= kDecConsumerWarps) return;
    for (int idx = threadIdx.x; idx < nh * D; idx += kDecConsumerWarps * 32) {
      const int hh = idx / D, dd = idx % D;
      const size_t row = static_cast<size_t>(b) * p.Hq + h0 + hh;
      if (p.splits == 1 && !p.partial_out) {
        p.out[row * D + dd] = __float2bfloat16(0.f);
        if (dd == 0 && p.lse) p.lse[row] = -INFINITY;
      } else {
        float* ws = p.ws + (row * p.splits + split) * Cfg::kPartialFloats;
        if (dd == 0) { ws[0] = -INFINITY; ws[1] = 0.f; ws[2] = 0.f; ws[3] = 0.f; }
        ws[4 + dd] = 0.f;
        ws[4 + D + dd] = 0.f;
      }
    }
    return;
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), kDecConsumerWarps);
    }
    fence_barrier_init();
  }
  __syncthreads();

  const int kvrow = b * p.Hkv + g;  // z coordinate of the 3-D tensor maps

  if (warp == kDecConsumerWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&vmap);
      bool ok = true;
      int issued = 0;
      for (int t = 0; t < ntiles; ++t) {
        const int s = t % NS;
        if (t >= NS) {
          if (!mbar_wait(smem_u32(&empty_bar[s]), ((t / NS) - 1) & 1, kErrDecodeEmpty)) { ok = false; break; }
        }
        const uint32_t fb = smem_u32(&full_bar[s]);
        mbar_arrive_expect_tx(fb, Cfg::kStageBytes);
        const uint32_t kdst = smem_u32(smem + s * Cfg::kStageBytes);
        const uint32_t vdst = kdst + Cfg::kTileBytes;
        const int key0 = kbeg + t * kDecTileKeys;
        if (!PAGED) {
#pragma unroll
          for (int hf = 0; hf < Cfg::kHalves; ++hf) {
            tma_load_3d(&kmap, kdst + hf * (kDecTileKeys * 128), fb, hf * 64, key0, kvrow);
            tma_load_3d(&vmap, vdst + hf * (kDecTileKeys * 128), fb, hf * 64, key0, kvrow);
          }
        } else {
          // one load per page part of the tile: plane = page * Hkv + g, row within the page
          for (int part = 0; part * p.box_rows < kDecTileKeys; ++part) {
            const int key = key0 + part * p.box_rows;
            int plane = 0, row = p.page_size;  // default: past the page, zero fill
            if (key < kend) {
              const int pg = __ldg(p.block_table + static_cast<size_t>(b) * p.max_pages + (key >> p.page_shift));
              if (pg >= 0 && pg < p.num_pages) {
                plane = pg * p.Hkv + g;
                row = key & (p.page_size - 1);
              }
            }
            const uint32_t off = static_cast<uint32_t>(part * p.box_rows * 128);
#pragma unroll
            for (int hf = 0; hf < Cfg::kHalves; ++hf) {
              tma_load_3d(&kmap, kdst + hf * (kDecTileKeys * 128) + off, fb, hf * 64, row, plane);
              tma_load_3d(&vmap, vdst + hf * (kDecTileKeys * 128) + off, fb, hf * 64, row, plane);
            }
          }
        }
        issued = t + 1;
      }
      if (!ok) {
        // Drain: every load issued must land before this CTA's smem goes away.
        for (int t = max(0, issued - NS); t < issued; ++t)
          mbar_wait(smem_u32(&full_bar[t % NS]), (t / NS) & 1, kErrDecodeDrain);
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int gr = lane >> 2;        // fragment row 0..7 -> query head h0 + gr
  const int qc = lane & 3;         // fragment column pair
  const bool live = gr < nh;
  const size_t qrow = static_cast<size_t>(b) * p.Hq + h0 + (live ? gr : 0);

  // Stacked A operand for the score MMA: rows 0..7 = q (scaled later in fp32),
  // rows 8..15 = rho; dead rows are zero.
  uint32_t afrag[D / 16][4];
  {
    const uint32_t* qv = reinterpret_cast<const uint32_t*>(p.q + qrow * D);
    const uint32_t* rv = HAS_R ? reinterpret_cast<const uint32_t*>(p.r + qrow * D) : nullptr;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      const int w0 = (ks * 16 + qc * 2) >> 1, w1 = (ks * 16 + 8 + qc * 2) >> 1;
      afrag[ks][0] = live ? __ldg(qv + w0) : 0u;
      afrag[ks][2] = live ? __ldg(qv + w1) : 0u;
      afrag[ks][1] = (HAS_R && live) ? __ldg(rv + w0) : 0u;
      afrag[ks][3] = (HAS_R && live) ? __ldg(rv + w1) : 0u;
    }
  }

  float o[D / 8][4];
#pragma unroll
  for (int j = 0; j < D / 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  // this thread's column share: l = sum p (fp32, also gives lse), c = sum of
  // the bf16-rounded p*s the value MMA consumes (so that O2 and c agree)
  float m_run = -INFINITY, l_run = 0.f, c_run = 0.f;

  // ldmatrix row addresses (relative to a K or V tile) for this lane.
  const int mi = lane >> 3, ri = lane & 7;
  const int kkey = warp * 16 + (mi >> 1) * 8 + ri;   // K: matrices (keys lo/hi) x (d lo/hi)
  const int vkey = warp * 16 + (mi & 1) * 8 + ri;    // V: matrices (keys lo/hi) x (d lo/hi), transposed
  bool ok = true;

  for (int t = 0; t < ntiles; ++t) {
    const int s = t % NS;
    // all lanes wait; the warp continues only if every lane saw the stage land
    const bool landed = mbar_wait(smem_u32(&full_bar[s]), (t / NS) & 1, kErrDecodeFull);
    if (!__all_sync(0xffffffffu, landed)) { ok = false; break; }
    const uint32_t kbase = smem_u32(smem + s * Cfg::kStageBytes);
    const uint32_t vbase = kbase + Cfg::kTileBytes;

    // ---- scores: acc[n] for keys n*8..n*8+7 of this warp's 16
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      const int chunk = (2 * ks + (mi & 1)) & 7;
      const uint32_t addr = kbase + (ks >> 2) * (kDecTileKeys * 128) + sw128(kkey, chunk);
      uint32_t b0, b1, b2, b3;
      ldsm_x4(addr, b0, b1, b2, b3);
      mma_bf16_16816(acc[0], afrag[ks], b0, b1);
      mma_bf16_16816(acc[1], afrag[ks], b2, b3);
    }

    // ---- shared online softmax over both branches
    const int key_lo = kbeg + t * kDecTileKeys + warp * 16 + qc * 2;  // key of acc[0][0]
    float x[4];
#pragma unroll
    for (int n = 0; n < 2; ++n)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int key = key_lo + n * 8 + e;
        x[n * 2 + e] = key < kend ? acc[n][e] * p.scale_log2 : -INFINITY;
      }
    float tmax = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
    const float m_new = fmaxf(m_run, tmax);
    const float m_use = m_new == -INFINITY ? 0.f : m_new;
    const float alpha = ex2(m_run - m_use);
    float pr[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) pr[i] = ex2(x[i] - m_use);
    const float sv[4] = {acc[0][2], acc[0][3], acc[1][2], acc[1][3]};  // rho.k, same keys
    float ps[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) ps[i] = HAS_R ? pr[i] * sv[i] : 0.f;
    // stacked A operand of the value MMA: rows g = P, rows g+8 = P*S (bf16)
    uint32_t pa[4];
    pa[0] = pack_bf16(pr[0], pr[1]);
    pa[1] = pack_bf16(ps[0], ps[1]);
    pa[2] = pack_bf16(pr[2], pr[3]);
    pa[3] = pack_bf16(ps[2], ps[3]);
    const float psum = (pr[0] + pr[1]) + (pr[2] + pr[3]);
    const float csum = (bf16_lo(pa[1]) + bf16_hi(pa[1])) + (bf16_lo(pa[3]) + bf16_hi(pa[3]));
    l_run = l_run * alpha + psum;
    c_run = c_run * alpha + csum;
    m_run = m_new;
    if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
      for (int j = 0; j < D / 8; ++j) {
        o[j][0] *= alpha; o[j][1] *= alpha; o[j][2] *= alpha; o[j][3] *= alpha;
      }
    }

    // ---- value product with the stacked [P ; P*S] operand
#pragma unroll
    for (int jp = 0; jp < D / 16; ++jp) {
      const int chunk = (2 * jp + (mi >> 1)) & 7;
      const uint32_t addr = vbase + (jp >> 2) * (kDecTileKeys * 128) + sw128(vkey, chunk);
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(addr, b0, b1, b2, b3);
      mma_bf16_16816(o[2 * jp], pa, b0, b1);
      mma_bf16_16816(o[2 * jp + 1], pa, b2, b3);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&empty_bar[s]));
  }

  // ---- merge the four warps' states through shared memory (stages are idle now)
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
  c_run += __shfl_xor_sync(0xffffffffu, c_run, 1);
  c_run += __shfl_xor_sync(0xffffffffu, c_run, 2);
  asm volatile("bar.sync 1, %0;" ::"n"(kDecConsumerWarps * 32) : "memory");

  constexpr int kRowF = 2 * D + 4;  // m, l, c, pad, O1[D], O2[D]
  float* red = reinterpret_cast<float*>(smem);
  {
    float* mine = red + (warp * 8 + gr) * kRowF;
    if (qc == 0) { mine[0] = m_run; mine[1] = l_run; mine[2] = c_run; mine[3] = 0.f; }
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
      const int dd = j * 8 + qc * 2;
      mine[4 + dd] = o[j][0];
      mine[4 + dd + 1] = o[j][1];
      mine[4 + D + dd] = o[j][2];
      mine[4 + D + dd + 1] = o[j][3];
    }
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kDecConsumerWarps * 32) : "memory");
  if (!ok) return;  // a wait ran out; the error word is set, results are undefined

  for (int idx = threadIdx.x; idx < nh * D; idx += kDecConsumerWarps * 32) {
    const int hh = idx / D, dd = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDecConsumerWarps; ++w) M = fmaxf(M, red[(w * 8 + hh) * kRowF]);
    const float Mu = M == -INFINITY ? 0.f : M;
    float L = 0.f, C = 0.f, O1 = 0.f, O2 = 0.f;
#pragma unroll
    for (int w = 0; w < kDecConsumerWarps; ++w) {
      const float* rw = red + (w * 8 + hh) * kRowF;
      const float beta = ex2(rw[0] - Mu);
      L += beta * rw[1];
      C += beta * rw[2];
      O1 += beta * rw[4 + dd];
      O2 += beta * rw[4 + D + dd];
    }
    const size_t row = static_cast<size_t>(b) * p.Hq + h0 + hh;
    if (p.splits == 1 && !p.partial_out) {
      float res = 0.f;
      if (L > 0.f) {
        const float inv = 1.f / L;
        const float o1 = O1 * inv;
        res = o1 - (O2 * inv - (C * inv) * o1);
      }
      p.out[row * D + dd] = __float2bfloat16(res);
      if (dd == 0 && p.lse) p.lse[row] = L > 0.f ? (M + __log2f(L)) * kLn2 : -INFINITY;
    } else {
      float* ws = p.ws + (row * p.splits + split) * Cfg::kPartialFloats;
      if (dd == 0) { ws[0] = M; ws[1] = L; ws[2] = C; ws[3] = 0.f; }
      ws[4 + dd] = O1;
      ws[4 + D + dd] = O2;
    }
  }
  // this CTA's results are written: the combine (launched as a programmatic
  // dependent) may be scheduled; it still waits for this grid to complete
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Merge the per-split partial states of one (b, h) row: one CTA of D threads.
template <int D>
__global__ void __launch_bounds__(D)
plx_decode_combine_kernel(const float* __restrict__ ws, __nv_bfloat16* __restrict__ out,
                          float* __restrict__ lse, int splits, int ranks, size_t rank_stride) {
  // partial states of row `row`: `ranks` blocks (rank_stride floats apart) of
  // `splits` consecutive states each; one block = one shard of the keys
  constexpr int PF = DecodeCfg<D>::kPartialFloats;
  const size_t row = blockIdx.x;
  const int dd = threadIdx.x;
  // launched as a programmatic dependent of the split kernel: wait until that
  // grid has completed and its writes are visible (a no-op otherwise)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  float M = -INFINITY;
  for (int rk = 0; rk < ranks; ++rk) {
    const float* base = ws + rk * rank_stride + row * splits * PF;
    for (int s = 0; s < splits; ++s) M = fmaxf(M, __ldg(base + s * PF));
  }
  const float Mu = M == -INFINITY ? 0.f : M;
  float L = 0.f, C = 0.f, O1 = 0.f, O2 = 0.f;
  for (int rk = 0; rk < ranks; ++rk) {
    const float* base = ws + rk * rank_stride + row * splits * PF;
    for (int s = 0; s < splits; ++s) {
      const float* ps = base + s * PF;
      const float beta = ex2(__ldg(ps) - Mu);
      L += beta * __ldg(ps + 1);
      C += beta * __ldg(ps + 2);
      O1 += beta * __ldg(ps + 4 + dd);
      O2 += beta * __ldg(ps + 4 + D + dd);
    }
  }
  float res = 0.f;
  if (L > 0.f) {
    const float inv = 1.f / L;
    const float o1 = O1 * inv;
    res = o1 - (O2 * inv - (C * inv) * o1);
  }
  out[row * D + dd] = __float2bfloat16(res);
  if (dd == 0 && lse) lse[row] = L > 0.f ? (M + __log2f(L)) * kLn2 : -INFINITY;
}

}  // namespace plx
