// plx_decode.cuh -- decode step of the Parallax forward pass, balanced over
// the key tiles of the whole batch.
//
// Work.  A segment is one (batch entry b, kv head g, group hg of <= 8 query
// heads): the query heads h0 .. h0 + nh - 1 of the group read the cached keys
// and values of (b, g) once (GQA packing).  Its live keys are cut into 64-key
// tiles.  The tiles of all segments, in the order (b, g, hg, tile), form one
// list, and a persistent grid of P CTAs takes it in equal contiguous ranges
// of tpc tiles (the last range may be shorter).  Every CTA therefore moves
// the same number of bytes whatever the sequence lengths are; a ragged batch
// leaves no CTA idle and no short sequence wastes a CTA.  The CTA finds the
// start of its range from the sequence lengths (a block-wide scan of the
// per-sequence tile counts) and walks the list from there.
//
// Pipeline.  A producer warp streams the K and V tiles with TMA into a
// 3-stage ring (6 at d = 64) with 128-byte swizzle; at the first tile of a
// segment it also copies the group's query and probe rows into the stage.
// The ring runs on across segment boundaries, so the next segment's tiles
// load while the current one finishes.  Four consumer warps take 16 keys of
// every tile each.
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
// Results.  At the last tile of a segment (or of its range) the four warps
// merge their states through the stage's shared memory.  A segment that the
// CTA covered whole is finished there: out = O1/l - (O2/l - (c/l)(O1/l)) and
// lse, or, for context parallelism, its state record.  A segment cut by a
// range boundary leaves one partial state (m, l, c, O1, O2) per CTA that
// touched it, and the combine kernel merges those, once the split grid is
// done: the CTA that began such a segment records where its partials are.
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
constexpr int kDecMinTilesPerCta = 4;   // smallest range: below this a CTA's ring has nothing to overlap
constexpr int kDecTailRows = 16;     // a sequence's last, partial tile is loaded in parts of this many keys
constexpr int kDecCombineThreads = 128;
constexpr int kCombineDepth = 4;  // partial states a combine warp has in flight

template <int D>
struct DecodeCfg {
  static constexpr int kHalves = D / 64;                       // 128-byte swizzle rows per key
  static constexpr int kTileBytes = kDecTileKeys * D * 2;      // one of K or V
  static constexpr int kKVBytes = 2 * kTileBytes;
  static constexpr int kQRBytes = 2 * 8 * D * 2;               // 8 query rows + 8 probe rows, bf16
  static constexpr int kStageBytes = kKVBytes + kQRBytes;      // a multiple of 1024
  static constexpr int kStages = D == 128 ? 3 : 6;
  static constexpr int kSmemBytes = kStages * kStageBytes + 1024 /*align*/ + 2 * kStages * 8 /*barriers*/;
  static constexpr int kChunkSmemBytes = kStages * kKVBytes + 1024 /*align*/ + 256 /*barriers*/;
  static constexpr int kRecFloats = 2 * D + 4;                 // m, l, c, pad, O1[D], O2[D]
  // the merge scratch of the four consumer warps fits in one stage:
  // O1, O2 of 8 rows in the K/V area, (m, l, c) in the query/probe area
  static_assert(kDecConsumerWarps * 8 * 2 * D * 4 <= kKVBytes, "merge scratch");
  static_assert(kDecConsumerWarps * 8 * 4 * 4 <= kQRBytes, "merge scratch");
  static_assert(kStageBytes % 1024 == 0, "stage alignment");
  static_assert((2 * kDecThreads + 4) * 4 <= kStageBytes, "partition scan scratch");
};

struct DecodeParams {
  const __nv_bfloat16* q;   // [B, Hq, D]
  const __nv_bfloat16* r;   // [B, Hq, D] or nullptr
  const int32_t* seqlens;   // [B]
  __nv_bfloat16* out;       // [B, Hq, D] (nullptr when rec_out)
  float* lse;               // [B, Hq] or nullptr
  float* rec_out;           // [B, Hq, 2D+4] state records instead of out (context parallel), or nullptr
  const int32_t* block_table;  // [B, max_pages] pool page of each page slot (paged caches)
  int num_pages, max_pages, page_size, page_shift, box_rows;  // paged caches: pool, table width, page
  float* ws;                // balanced plan: partial slots [2 * P][rps][2D+4] (slot 2c = CTA c's first
                            //   segment, 2c+1 its last); chunked plan: [B, Hq, splits, 2D+4]
  int chunk_tiles, splits;  // chunked plan: tiles per part and parts per segment (chunk_tiles 0: balanced plan)
  int B, Hq, Hkv, S_max, G, n_hgroups, rps;  // rps = min(G, 8) rows per partial slot
  int key_offset;           // global index of the cache's first key (context parallel; else 0)
  float scale_log2;         // scale * log2(e)
};

// Byte offset of (key row, 16-byte chunk) inside one 64-key x 128-byte block
// written by TMA with CU_TENSOR_MAP_SWIZZLE_128B.
__device__ __forceinline__ uint32_t sw128(int row, int chunk) {
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

// Live keys of sequence b in this cache (its keys past key_offset, at most S_max).
__device__ __forceinline__ int dec_live(const DecodeParams& p, int b) {
  const int n = __ldg(p.seqlens + b) - p.key_offset;
  return n < 0 ? 0 : (n > p.S_max ? p.S_max : n);
}
__device__ __forceinline__ int dec_ntiles(const DecodeParams& p, int b) {
  return (dec_live(p, b) + kDecTileKeys - 1) / kDecTileKeys;
}

// Non-tensor bulk copy global -> this CTA's shared memory, completion on `bar`
// (addresses 16-byte aligned, size a multiple of 16).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
               : "memory");
}

// Consumer: o += [P ; P*S] V over this warp's 16 keys of the stage's V tile
// (transposed ldmatrix: b0 / b2 hold keys qc*2, qc*2+1 of the first eight,
// b1 / b3 the same of the second eight, lower key in the low half).
template <int D, int TK = kDecTileKeys>
__device__ __forceinline__ void value_mma(float (&o)[D / 8][4], const uint32_t (&pa)[4], uint32_t vbase, int vkey,
                                          int mi) {
#pragma unroll
  for (int jp = 0; jp < D / 16; ++jp) {
    const int chunk = (2 * jp + (mi >> 1)) & 7;
    const uint32_t addr = vbase + (jp >> 2) * (TK * 128) + sw128(vkey, chunk);
    uint32_t b0, b1, b2, b3;
    ldsm_x4_t(addr, b0, b1, b2, b3);
    mma_bf16_16816(o[2 * jp], pa, b0, b1);
    mma_bf16_16816(o[2 * jp + 1], pa, b2, b3);
  }
}

// The same with the value rows of keys >= kend zeroed in the fragments, so
// that a zero weight times whatever those rows hold (Inf, NaN) adds nothing.
// key_lo = the key of this thread's first fragment element.
template <int D, int TK = kDecTileKeys>
__device__ __forceinline__ void value_mma_masked(float (&o)[D / 8][4], const uint32_t (&pa)[4], uint32_t vbase,
                                                 int vkey, int mi, int key_lo, int kend) {
  const uint32_t m_lo = (key_lo < kend ? 0x0000ffffu : 0u) | (key_lo + 1 < kend ? 0xffff0000u : 0u);
  const uint32_t m_hi = (key_lo + 8 < kend ? 0x0000ffffu : 0u) | (key_lo + 9 < kend ? 0xffff0000u : 0u);
#pragma unroll
  for (int jp = 0; jp < D / 16; ++jp) {
    const int chunk = (2 * jp + (mi >> 1)) & 7;
    const uint32_t addr = vbase + (jp >> 2) * (TK * 128) + sw128(vkey, chunk);
    uint32_t b0, b1, b2, b3;
    ldsm_x4_t(addr, b0, b1, b2, b3);
    b0 &= m_lo; b1 &= m_hi; b2 &= m_lo; b3 &= m_hi;
    mma_bf16_16816(o[2 * jp], pa, b0, b1);
    mma_bf16_16816(o[2 * jp + 1], pa, b2, b3);
  }
}

// Producer: the K and V tile of keys key0 .. key0 + 63 of plane kvrow into
// kdst / vdst (128-byte swizzled, D / 64 column halves of 64 rows each),
// completing on `bar`, which also expects `extra` bytes of other copies.  A
// tile with fewer than 64 live keys (the sequence's last) is loaded in
// kDecTailRows-key parts through the maps kmap_t / vmap_t, only as far as the
// live keys reach: the rows past them keep whatever the stage held before,
// which the consumers mask out.  A part's 16 x 128-byte boxes start on 2 KB
// boundaries, so the swizzle pattern of every row is the full tile's.
template <int D, int TK = kDecTileKeys>
__device__ __forceinline__ void load_kv_tile(const CUtensorMap* kmap, const CUtensorMap* vmap, const CUtensorMap* kmap_t,
                                             const CUtensorMap* vmap_t, uint32_t kdst, uint32_t vdst, uint32_t bar,
                                             int key0, int live_from_key0, int kvrow, uint32_t extra) {
  constexpr int kHalves = D / 64;
  if (live_from_key0 >= TK) {
    mbar_arrive_expect_tx(bar, 2u * TK * D * 2 + extra);
#pragma unroll
    for (int hf = 0; hf < kHalves; ++hf) {
      tma_load_3d(kmap, kdst + hf * (TK * 128), bar, hf * 64, key0, kvrow);
      tma_load_3d(vmap, vdst + hf * (TK * 128), bar, hf * 64, key0, kvrow);
    }
    return;
  }
  const int parts = (live_from_key0 + kDecTailRows - 1) / kDecTailRows;  // 1 .. 4
  mbar_arrive_expect_tx(bar, static_cast<uint32_t>(parts) * (2u * kDecTailRows * D * 2) + extra);
  for (int part = 0; part < parts; ++part) {
    const uint32_t off = static_cast<uint32_t>(part * kDecTailRows * 128);
#pragma unroll
    for (int hf = 0; hf < kHalves; ++hf) {
      tma_load_3d(kmap_t, kdst + hf * (TK * 128) + off, bar, hf * 64, key0 + part * kDecTailRows, kvrow);
      tma_load_3d(vmap_t, vdst + hf * (TK * 128) + off, bar, hf * 64, key0 + part * kDecTailRows, kvrow);
    }
  }
}

// Position in the tile list: segment (b, j = g * n_hgroups + hg), tile i of
// nb, with `live` keys in sequence b.
struct DecCursor {
  int b, j, i, nb, live;
  __device__ __forceinline__ void set_b(const DecodeParams& p, int bb) {
    b = bb;
    live = bb < p.B ? dec_live(p, bb) : kDecTileKeys;
    nb = (live + kDecTileKeys - 1) / kDecTileKeys;
  }
  __device__ __forceinline__ void advance(const DecodeParams& p, int HN) {
    if (++i < nb) return;
    i = 0;
    if (++j < HN) return;
    j = 0;
    // next sequence with live keys (past the last one, b = B stops the walk)
    do {
      set_b(p, b + 1);
    } while (nb == 0);
  }
};

// ---- where the work partitions fall in the tile list (shared by the split
// and the combine kernel, which computes the same plan independently)

// Block-wide: NT threads sum the tile counts of contiguous chunks of the
// batch; scratch[0..NT) = the sums, [NT..2NT) = their exclusive prefix,
// scratch[2NT] = the total (tiles of one segment of every sequence).
template <int NT>
__device__ __forceinline__ void dec_scan(const DecodeParams& p, int* scratch) {
  const int tid = threadIdx.x, lane = tid & 31;
  {
    const int per = (p.B + NT - 1) / NT;
    const int lo = tid * per, hi = min(p.B, lo + per);
    int sum = 0;
    for (int b = lo; b < hi; ++b) sum += dec_ntiles(p, b);
    scratch[tid] = sum;
  }
  __syncthreads();
  if (tid < 32) {
    constexpr int E = (NT + 31) / 32;  // entries per lane
    int v[E], lsum = 0;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int idx = lane * E + e;
      v[e] = idx < NT ? scratch[idx] : 0;
      lsum += v[e];
    }
    int incl = lsum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    int run = incl - lsum;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int idx = lane * E + e;
      if (idx < NT) scratch[NT + idx] = run;
      run += v[e];
    }
    if (lane == 31) scratch[2 * NT] = incl;
  }
  __syncthreads();
}

// Block-wide, after dec_scan: the sequence b whose segments hold list tile
// t (prefix(b) * HN <= t < prefix(b+1) * HN) goes to scratch[2NT+1] and
// prefix(b) to scratch[2NT+2].  Ends with a barrier.
template <int NT>
__device__ __forceinline__ void dec_find(const DecodeParams& p, int* scratch, int t, int HN) {
  const int tid = threadIdx.x;
  const int u = t / HN;
  const int part = scratch[tid], pre = scratch[NT + tid];
  if (part > 0 && pre <= u && u < pre + part) {
    const int per = (p.B + NT - 1) / NT;
    int acc = pre;
    for (int b = tid * per; b < min(p.B, (tid + 1) * per); ++b) {
      const int n = dec_ntiles(p, b);
      if (u < acc + n) {
        scratch[2 * NT + 1] = b;
        scratch[2 * NT + 2] = acc;
        break;
      }
      acc += n;
    }
  }
  __syncthreads();
}

// Tiles per partition: equal ranges, but at least kDecMinTilesPerCta.
__device__ __forceinline__ int dec_tpc(int T, int P) { return max((T + P - 1) / P, kDecMinTilesPerCta); }

template <int D, bool HAS_R, bool PAGED>
__global__ void __launch_bounds__(kDecThreads, 2)
plx_decode_split_kernel(const __grid_constant__ CUtensorMap kmap,
                        const __grid_constant__ CUtensorMap vmap,
                        const __grid_constant__ CUtensorMap kmap_t,
                        const __grid_constant__ CUtensorMap vmap_t, const DecodeParams p) {
  using Cfg = DecodeCfg<D>;
  constexpr int NS = Cfg::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + NS * Cfg::kStageBytes);
  uint64_t* empty_bar = full_bar + NS;

  // the combine kernel (a programmatic dependent) may be scheduled now; it
  // waits for this whole grid to complete before it reads anything we write
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int c = blockIdx.x;
  const int HN = p.Hkv * p.n_hgroups;

  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), kDecConsumerWarps);
    }
    fence_barrier_init();
  }
  if (tid == kDecConsumerWarps * 32) {
    // the descriptors' fetch overlaps the range search below
    tma_prefetch_desc(&kmap);
    tma_prefetch_desc(&vmap);
    tma_prefetch_desc(&kmap_t);
    tma_prefetch_desc(&vmap_t);
  }
  // ---- this CTA's range of the tile list (scratch: stage 0, before any load)
  int* scratch = reinterpret_cast<int*>(smem);
  DecCursor cur;
  int t_begin, t_end, tpc = 0;
  {
    // balanced plan: CTA c takes tiles [c tpc, (c+1) tpc) of the batch's tile list
    // (scratch: stage 0, before any load)
    int* scratch = reinterpret_cast<int*>(smem);
    dec_scan<kDecThreads>(p, scratch);
    const int T = scratch[2 * kDecThreads] * HN;  // tiles in the whole list
    tpc = dec_tpc(T, gridDim.x);
    t_begin = c * tpc;
    if (t_begin >= T) return;  // uniform: the whole CTA has no tiles
    t_end = min(t_begin + tpc, T);
    dec_find<kDecThreads>(p, scratch, t_begin, HN);
    cur.set_b(p, scratch[2 * kDecThreads + 1]);
    const int local = t_begin - scratch[2 * kDecThreads + 2] * HN;
    cur.j = local / cur.nb;
    cur.i = local % cur.nb;
    // every thread has read the scratch: stage 0 may be loaded (the proxy fence
    // orders the scratch writes before the TMA writes to the same bytes)
    fence_proxy_async_smem();
    __syncthreads();
  }

  if (warp == kDecConsumerWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      bool ok = true;
      int k = 0;  // tiles issued
      for (int t = t_begin; t < t_end && ok;) {
        const int n = min(cur.nb - cur.i, t_end - t);  // tiles of this segment in the range
        const int g = cur.j / p.n_hgroups, hg = cur.j % p.n_hgroups;
        const int nh = min(8, p.G - hg * 8);
        const int kvrow = cur.b * p.Hkv + g;  // z coordinate of the 3-D tensor maps
        const uint32_t qr_bytes = static_cast<uint32_t>((HAS_R ? 2 : 1) * nh * D * 2);
        for (int u = 0; u < n; ++u, ++k) {
          const int s = k % NS;
          if (k >= NS && !mbar_wait(smem_u32(&empty_bar[s]), ((k / NS) - 1) & 1, kErrDecodeEmpty)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&full_bar[s]);
          const uint32_t kdst = smem_u32(smem + s * Cfg::kStageBytes);
          const uint32_t vdst = kdst + Cfg::kTileBytes;
          const int key0 = (cur.i + u) * kDecTileKeys;
          if (!PAGED) {
            load_kv_tile<D>(&kmap, &vmap, &kmap_t, &vmap_t, kdst, vdst, fb, key0, cur.live - key0, kvrow,
                            u == 0 ? qr_bytes : 0u);
          } else {
            mbar_arrive_expect_tx(fb, Cfg::kKVBytes + (u == 0 ? qr_bytes : 0u));
            // one load per page part of the tile: plane = page * Hkv + g, row within the page
            for (int part = 0; part * p.box_rows < kDecTileKeys; ++part) {
              const int key = key0 + part * p.box_rows;
              int plane = 0, row = p.page_size;  // default: past the page, zero fill
              if (key < cur.live) {
                const int pg = __ldg(p.block_table + static_cast<size_t>(cur.b) * p.max_pages + (key >> p.page_shift));
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
          if (u == 0) {
            const size_t row0 = static_cast<size_t>(cur.b) * p.Hq + g * p.G + hg * 8;
            const uint32_t qdst = kdst + Cfg::kKVBytes;
            bulk_load(qdst, p.q + row0 * D, nh * D * 2, fb);
            if (HAS_R) bulk_load(qdst + 8 * D * 2, p.r + row0 * D, nh * D * 2, fb);
          }
        }
        t += n;
        cur.i += n - 1;
        cur.advance(p, HN);
      }
      // Drain: every load issued must land before this CTA's shared memory
      // goes away (the consumers stop waiting once a wait has run out).
      for (int j = max(0, k - NS); j < k; ++j)
        mbar_wait(smem_u32(&full_bar[j % NS]), (j / NS) & 1, kErrDecodeDrain);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int gr = lane >> 2;        // fragment row 0..7 -> query head h0 + gr
  const int qc = lane & 3;         // fragment column pair
  const int mi = lane >> 3, ri = lane & 7;
  const int kkey = warp * 16 + (mi >> 1) * 8 + ri;   // K: matrices (keys lo/hi) x (d lo/hi)
  const int vkey = warp * 16 + (mi & 1) * 8 + ri;    // V: matrices (keys lo/hi) x (d lo/hi), transposed
  bool ok = true;

  // Control flow is the same for every consumer warp whatever happens: a warp
  // whose wait runs out (or that sees another CTA's error) stops waiting but
  // goes on through the loop (its shared-memory reads and global writes stay
  // in bounds) and takes every named barrier below, so no warp is left
  // waiting at one; the results are then undefined (the error word is set).
  int k = 0;  // tiles consumed
  for (int t = t_begin; t < t_end;) {
    const int n = min(cur.nb - cur.i, t_end - t);  // tiles of this segment in the range
    const int g = cur.j / p.n_hgroups, hg = cur.j % p.n_hgroups;
    const int nh = min(8, p.G - hg * 8);
    const bool live = gr < nh;
    const int kend = cur.live;
    const int i0 = cur.i;

    uint32_t afrag[D / 16][4];
    float o[D / 8][4];
#pragma unroll
    for (int jj = 0; jj < D / 8; ++jj) o[jj][0] = o[jj][1] = o[jj][2] = o[jj][3] = 0.f;
    // this thread's column share: l = sum p (fp32, also gives lse), c = sum of
    // the bf16-rounded p*s the value MMA consumes (so that O2 and c agree)
    float m_run = -INFINITY, l_run = 0.f, c_run = 0.f;

    for (int u = 0; u < n; ++u, ++k) {
      const int s = k % NS;
      const bool landed = ok && mbar_wait(smem_u32(&full_bar[s]), (k / NS) & 1, kErrDecodeFull);
      ok = __all_sync(0xffffffffu, landed);
      uint8_t* stage = smem + s * Cfg::kStageBytes;
      const uint32_t kbase = smem_u32(stage);
      const uint32_t vbase = kbase + Cfg::kTileBytes;
      if (u == 0) {
        // stacked A operand of the score MMA: rows 0..7 = q (scaled later in
        // fp32), rows 8..15 = rho; rows past the group are zero
        const uint32_t* qs = reinterpret_cast<const uint32_t*>(stage + Cfg::kKVBytes) + gr * (D / 2);
        const uint32_t* rs = qs + 8 * (D / 2);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const int w0 = (ks * 16 + qc * 2) >> 1, w1 = (ks * 16 + 8 + qc * 2) >> 1;
          afrag[ks][0] = live ? qs[w0] : 0u;
          afrag[ks][2] = live ? qs[w1] : 0u;
          afrag[ks][1] = (HAS_R && live) ? rs[w0] : 0u;
          afrag[ks][3] = (HAS_R && live) ? rs[w1] : 0u;
        }
      }

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
      const int key_lo = (i0 + u) * kDecTileKeys + warp * 16 + qc * 2;  // key of acc[0][0]
      // Keys past the sequence (the tail of its last tile) take no part,
      // whatever their rows hold: -inf scores, zero rho.k, zero value rows.
      float x[4], sv[4];
#pragma unroll
      for (int nn = 0; nn < 2; ++nn)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const bool in = key_lo + nn * 8 + e < kend;
          x[nn * 2 + e] = in ? acc[nn][e] * p.scale_log2 : -INFINITY;
          sv[nn * 2 + e] = in ? acc[nn][2 + e] : 0.f;  // rho.k, same keys
        }
      float tmax = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
      tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
      tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
      const float m_new = fmaxf(m_run, tmax);
      const float m_use = m_new == -INFINITY ? 0.f : m_new;
      const float alpha = ex2(m_run - m_use);
      float pr[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) pr[e] = ex2(x[e] - m_use);
      float ps[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) ps[e] = HAS_R ? pr[e] * sv[e] : 0.f;
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
        for (int jj = 0; jj < D / 8; ++jj) {
          o[jj][0] *= alpha; o[jj][1] *= alpha; o[jj][2] *= alpha; o[jj][3] *= alpha;
        }
      }

      // ---- value product with the stacked [P ; P*S] operand
      if (key_lo - qc * 2 + 16 <= kend)  // warp-uniform: all 16 keys of this warp are live
        value_mma<D>(o, pa, vbase, vkey, mi);
      else
        value_mma_masked<D>(o, pa, vbase, vkey, mi, key_lo, kend);
      if (u + 1 < n) {
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&empty_bar[s]));
      }
    }

    // ---- merge the four warps' states through the last tile's stage
    const int s = (k - 1) % NS;
    uint8_t* stage = smem + s * Cfg::kStageBytes;
    float l4 = l_run, c4 = c_run;
    l4 += __shfl_xor_sync(0xffffffffu, l4, 1);
    l4 += __shfl_xor_sync(0xffffffffu, l4, 2);
    c4 += __shfl_xor_sync(0xffffffffu, c4, 1);
    c4 += __shfl_xor_sync(0xffffffffu, c4, 2);
    asm volatile("bar.sync 1, %0;" ::"n"(kDecConsumerWarps * 32) : "memory");  // every warp is done with K/V
    float* sc = reinterpret_cast<float*>(stage);                        // [warp][row][2D], swizzled columns
    float* mlc = reinterpret_cast<float*>(stage + Cfg::kKVBytes);       // [warp][row][4]
    if (live) {  // rows past the group hold nothing
      const int swz = (gr & 3) << 3;
      float* mine = sc + (warp * 8 + gr) * (2 * D);
      if (qc == 0) {
        float* h = mlc + (warp * 8 + gr) * 4;
        h[0] = m_run; h[1] = l4; h[2] = c4;
      }
#pragma unroll
      for (int jj = 0; jj < D / 8; ++jj) {
        const int col = (jj * 8 + qc * 2) ^ swz;
        *reinterpret_cast<float2*>(mine + col) = make_float2(o[jj][0], o[jj][1]);
        *reinterpret_cast<float2*>(mine + D + col) = make_float2(o[jj][2], o[jj][3]);
      }
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kDecConsumerWarps * 32) : "memory");
    const int h0 = g * p.G + hg * 8;
    // a segment this CTA covered whole is finished here; otherwise the state goes to its slot
    const bool whole = i0 == 0 && n == cur.nb;
    const int slot = t == t_begin ? 2 * c : 2 * c + 1;
    for (int idx = tid; idx < nh * D; idx += kDecConsumerWarps * 32) {
      const int hh = idx / D, dd = idx % D;
      const int col = dd ^ ((hh & 3) << 3);
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kDecConsumerWarps; ++w) M = fmaxf(M, mlc[(w * 8 + hh) * 4]);
      const float Mu = M == -INFINITY ? 0.f : M;
      float L = 0.f, C = 0.f, O1 = 0.f, O2 = 0.f;
#pragma unroll
      for (int w = 0; w < kDecConsumerWarps; ++w) {
        const float* hw = mlc + (w * 8 + hh) * 4;
        const float* rw = sc + (w * 8 + hh) * (2 * D);
        const float beta = ex2(hw[0] - Mu);
        L += beta * hw[1];
        C += beta * hw[2];
        O1 += beta * rw[col];
        O2 += beta * rw[D + col];
      }
      const size_t row = static_cast<size_t>(cur.b) * p.Hq + h0 + hh;
      float* rec = nullptr;
      if (!whole) rec = p.ws + (static_cast<size_t>(slot) * p.rps + hh) * Cfg::kRecFloats;
      else if (p.rec_out) rec = p.rec_out + row * Cfg::kRecFloats;
      if (rec) {
        if (dd == 0) { rec[0] = M; rec[1] = L; rec[2] = C; rec[3] = 0.f; }
        rec[4 + dd] = O1;
        rec[4 + D + dd] = O2;
      } else {
        float res = 0.f;
        if (L > 0.f) {
          const float inv = 1.f / L;
          const float o1 = O1 * inv;
          res = o1 - (O2 * inv - (C * inv) * o1);
        }
        p.out[row * D + dd] = __float2bfloat16(res);
        if (dd == 0 && p.lse) p.lse[row] = L > 0.f ? (M + __log2f(L)) * kLn2 : -INFINITY;
      }
    }
    // the scratch is read; generic writes must be ordered before the next TMA into this stage
    fence_proxy_async_smem();
    asm volatile("bar.sync 1, %0;" ::"n"(kDecConsumerWarps * 32) : "memory");
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&empty_bar[s]));
    t += n;
    cur.i += n - 1;
    cur.advance(p, HN);
  }
}

// The chunked plan: one CTA per (chunk `split` of chunk_tiles tiles, kv head
// and head group, batch entry b) -- the grid is (splits, Hkv * n_hgroups, B).
// Same per-tile work as the balanced kernel; the chunk's partial state goes to
// [B, Hq, splits, 2D+4] (or, with one chunk per segment, the output itself)
// and plx_record_merge_kernel merges the chunks of every row.
template <int D, bool HAS_R, bool PAGED>
__global__ void __launch_bounds__(kDecThreads, 2)
plx_decode_chunk_kernel(const __grid_constant__ CUtensorMap kmap,
                        const __grid_constant__ CUtensorMap vmap,
                        const __grid_constant__ CUtensorMap kmap_t,
                        const __grid_constant__ CUtensorMap vmap_t, const DecodeParams p) {
  using Cfg = DecodeCfg<D>;
  constexpr int NS = Cfg::kStages;
  constexpr int kStride = Cfg::kKVBytes;  // stage stride: K and V tiles only
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + NS * kStride);
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
  const int chunk = p.chunk_tiles * kDecTileKeys;
  const int kbeg = split * chunk;
  const int kend = min(kbeg + chunk, seqlen);
  const int ntiles = kend > kbeg ? (kend - kbeg + kDecTileKeys - 1) / kDecTileKeys : 0;

  if (ntiles == 0) {
    // Empty chunk: an empty partial state, or (single split) the empty-set output.
    if (warp >= kDecConsumerWarps) return;
    for (int idx = threadIdx.x; idx < nh * D; idx += kDecConsumerWarps * 32) {
      const int hh = idx / D, dd = idx % D;
      const size_t row = static_cast<size_t>(b) * p.Hq + h0 + hh;
      if (p.splits == 1) {
        p.out[row * D + dd] = __float2bfloat16(0.f);
        if (dd == 0 && p.lse) p.lse[row] = -INFINITY;
      } else {
        float* ws = p.ws + (row * p.splits + split) * Cfg::kRecFloats;
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
        const uint32_t kdst = smem_u32(smem + s * kStride);
        const uint32_t vdst = kdst + Cfg::kTileBytes;
        const int key0 = kbeg + t * kDecTileKeys;
        if (!PAGED) {
          load_kv_tile<D>(&kmap, &vmap, &kmap_t, &vmap_t, kdst, vdst, fb, key0, kend - key0, kvrow, 0u);
        } else {
          mbar_arrive_expect_tx(fb, kStride);
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
    const uint32_t kbase = smem_u32(smem + s * kStride);
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
    // keys past the sequence take no part, whatever their rows hold
    float x[4], sv[4];
#pragma unroll
    for (int n = 0; n < 2; ++n)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const bool in = key_lo + n * 8 + e < kend;
        x[n * 2 + e] = in ? acc[n][e] * p.scale_log2 : -INFINITY;
        sv[n * 2 + e] = in ? acc[n][2 + e] : 0.f;  // rho.k, same keys
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
    if (key_lo - qc * 2 + 16 <= kend)  // warp-uniform: all 16 keys of this warp are live
      value_mma<D>(o, pa, vbase, vkey, mi);
    else
      value_mma_masked<D>(o, pa, vbase, vkey, mi, key_lo, kend);
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
    if (p.splits == 1) {
      float res = 0.f;
      if (L > 0.f) {
        const float inv = 1.f / L;
        const float o1 = O1 * inv;
        res = o1 - (O2 * inv - (C * inv) * o1);
      }
      p.out[row * D + dd] = __float2bfloat16(res);
      if (dd == 0 && p.lse) p.lse[row] = L > 0.f ? (M + __log2f(L)) * kLn2 : -INFINITY;
    } else {
      float* ws = p.ws + (row * p.splits + split) * Cfg::kRecFloats;
      if (dd == 0) { ws[0] = M; ws[1] = L; ws[2] = C; ws[3] = 0.f; }
      ws[4 + dd] = O1;
      ws[4 + D + dd] = O2;
    }
  }
  // this CTA's results are written: the combine (launched as a programmatic
  // dependent) may be scheduled; it still waits for this grid to complete
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---- the segment plan: many short streams.  Each of the W warps of a CTA
// owns whole segments and streams their keys through a ring of its own in
// TK-key stages, its lane 0 issuing the TMA loads of the stage it just
// finished (loads run on across the warp's segment boundaries).  Segments
// are dealt round the CTAs first (segment k goes to CTA k mod P, warp
// (k div P) mod W), so a batch with few segments still spreads over the
// SMs.  A warp holds a segment's whole online state, so a segment ends with
// quad shuffles and direct stores: no cross-warp merge, no partial states,
// one kernel.  The next segment's query and probe rows are fetched into
// registers while the current one streams.  Two shapes share the code: 4
// warps with 32-key stages (more bytes in flight per warp, for fewer
// segments) and 8 warps with 16-key stages (two warps per sub-partition to
// hide each other's latencies, for many); both keep 192 KB of stages per SM.
template <int D, int W, int TK>
struct SegCfg {
  static constexpr int kThreads = W * 32;
  static constexpr int kTileBytes = TK * D * 2;             // one of K or V
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kStages = (D == 128 ? 3 : 6) * 32 / (TK * (W / 4));  // per warp
  static constexpr int kWarpBytes = kStages * kStageBytes;
  static constexpr int kSmemBytes = W * kWarpBytes + 1024 + W * kStages * 8;
  static_assert(kStages >= 2, "a ring of at least two stages per warp");
  static_assert(kStageBytes % 1024 == 0, "stage alignment");
  static_assert(kSmemBytes <= 227 * 1024, "one CTA per SM");
};
constexpr int kSegFewWarps = 4, kSegFewKeys = 32;   // shape for fewer segments
constexpr int kSegManyWarps = 8, kSegManyKeys = 16; // shape for many segments

// Position in one warp's segment stream: segment sg (of `total`), tile t of nt.
template <int TK>
struct SegWalk {
  int sg, t, nt, live, total, stride;
  __device__ __forceinline__ void set(const DecodeParams& p, int HN) {
    nt = 0;
    live = 0;
    if (sg < total) {
      live = dec_live(p, sg / HN);
      nt = (live + TK - 1) / TK;
    }
  }
  // first tile at or after segment sg (skipping segments with no live key); false past the end
  __device__ __forceinline__ bool seek(const DecodeParams& p, int HN) {
    for (;;) {
      if (sg >= total) return false;
      set(p, HN);
      if (nt > 0) { t = 0; return true; }
      sg += stride;
    }
  }
  __device__ __forceinline__ bool next(const DecodeParams& p, int HN) {
    if (++t < nt) return true;
    sg += stride;
    return seek(p, HN);
  }
};

// q (rows 0..7) and rho (rows 8..15) of segment sg as the stacked A fragments
// of the score MMA; rows past the group are zero
template <int D, bool HAS_R>
__device__ __forceinline__ void seg_load_qr(const DecodeParams& p, int sg, int HN, uint32_t (&af)[D / 16][4]) {
  const int lane = threadIdx.x & 31, gr = lane >> 2, qc = lane & 3;
  const int b = sg / HN, j = sg % HN;
  const int g = j / p.n_hgroups, hg = j % p.n_hgroups;
  const int nh = min(8, p.G - hg * 8);
  const bool live = gr < nh;
  const size_t row = static_cast<size_t>(b) * p.Hq + g * p.G + hg * 8 + (live ? gr : 0);
  const uint32_t* qv = reinterpret_cast<const uint32_t*>(p.q + row * D);
  const uint32_t* rv = HAS_R ? reinterpret_cast<const uint32_t*>(p.r + row * D) : nullptr;
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    const int w0 = (ks * 16 + qc * 2) >> 1, w1 = (ks * 16 + 8 + qc * 2) >> 1;
    af[ks][0] = live ? __ldg(qv + w0) : 0u;
    af[ks][2] = live ? __ldg(qv + w1) : 0u;
    af[ks][1] = (HAS_R && live) ? __ldg(rv + w0) : 0u;
    af[ks][3] = (HAS_R && live) ? __ldg(rv + w1) : 0u;
  }
}

template <int D, bool HAS_R, int W, int TK>
__global__ void __launch_bounds__(W * 32, 1)
plx_decode_seg_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                      const __grid_constant__ CUtensorMap kmap_t, const __grid_constant__ CUtensorMap vmap_t,
                      const DecodeParams p) {
  using Cfg = SegCfg<D, W, TK>;
  constexpr int NS = Cfg::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* ring = smem + warp * Cfg::kWarpBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + W * Cfg::kWarpBytes) + warp * NS;
  const int HN = p.Hkv * p.n_hgroups;

  if (lane == 0) {
    for (int s = 0; s < NS; ++s) mbar_init(smem_u32(&full[s]), 1);
    fence_barrier_init();
    tma_prefetch_desc(&kmap);
    tma_prefetch_desc(&vmap);
    tma_prefetch_desc(&kmap_t);
    tma_prefetch_desc(&vmap_t);
  }
  __syncwarp();

  const int stride = gridDim.x * W;
  const int first = warp * gridDim.x + blockIdx.x;
  // lane 0's load cursor: the first NS tiles of this warp's stream
  SegWalk<TK> ld{first, 0, 0, 0, p.B * HN, stride};
  int issued = 0;
  bool more = false;
  auto issue = [&](int s) {
    const uint32_t kdst = smem_u32(ring + s * Cfg::kStageBytes);
    const int b = ld.sg / HN, g = (ld.sg % HN) / p.n_hgroups;
    load_kv_tile<D, TK>(&kmap, &vmap, &kmap_t, &vmap_t, kdst, kdst + Cfg::kTileBytes, smem_u32(&full[s]),
                        ld.t * TK, ld.live - ld.t * TK, b * p.Hkv + g, 0u);
  };
  if (lane == 0) {
    more = ld.seek(p, HN);
    while (more && issued < NS) {
      issue(issued % NS);
      ++issued;
      more = ld.next(p, HN);
    }
  }

  const int gr = lane >> 2, qc = lane & 3;
  const int mi = lane >> 3, ri = lane & 7;
  bool ok = true;
  int k = 0;  // tiles consumed
  uint32_t afn[D / 16][4];
  if (first < p.B * HN) seg_load_qr<D, HAS_R>(p, first, HN, afn);
  for (int sg = first; sg < p.B * HN && ok; sg += stride) {
    uint32_t afrag[D / 16][4];
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks)
#pragma unroll
      for (int e = 0; e < 4; ++e) afrag[ks][e] = afn[ks][e];
    if (sg + stride < p.B * HN) seg_load_qr<D, HAS_R>(p, sg + stride, HN, afn);  // in flight while this streams
    const int b = sg / HN, j = sg % HN;
    const int g = j / p.n_hgroups, hg = j % p.n_hgroups;
    const int nh = min(8, p.G - hg * 8);
    const size_t row0 = static_cast<size_t>(b) * p.Hq + g * p.G + hg * 8;
    const int kend = dec_live(p, b);
    const int nt = (kend + TK - 1) / TK;
    if (nt == 0) {
      // no live key: out = 0, lse = -inf (or an empty record)
      if (p.rec_out) {
        for (int idx = lane; idx < nh * (2 * D + 4); idx += 32)
          p.rec_out[row0 * (2 * D + 4) + idx] = (idx % (2 * D + 4)) == 0 ? -INFINITY : 0.f;
      } else {
        for (int idx = lane; idx < nh * D; idx += 32) p.out[row0 * D + idx] = __float2bfloat16(0.f);
        if (p.lse && lane < nh) p.lse[row0 + lane] = -INFINITY;
      }
      continue;
    }

    float o[D / 8][4];
#pragma unroll
    for (int jj = 0; jj < D / 8; ++jj) o[jj][0] = o[jj][1] = o[jj][2] = o[jj][3] = 0.f;
    float m_run = -INFINITY, l_run = 0.f, c_run = 0.f;
    for (int t = 0; t < nt; ++t, ++k) {
      const int s = k % NS;
      // a wait that runs out stops this warp (its results are then undefined;
      // the error word is set); no other warp waits for it
      const bool landed = mbar_wait(smem_u32(&full[s]), (k / NS) & 1, kErrDecodeFull);
      if (!__all_sync(0xffffffffu, landed)) { ok = false; break; }
      const uint32_t kbase = smem_u32(ring + s * Cfg::kStageBytes);
      const uint32_t vbase = kbase + Cfg::kTileBytes;
#pragma unroll
      for (int s16 = 0; s16 < TK / 16; ++s16) {
        const int kkey = s16 * 16 + (mi >> 1) * 8 + ri;
        const int vkey = s16 * 16 + (mi & 1) * 8 + ri;
        float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const int chunk = (2 * ks + (mi & 1)) & 7;
          const uint32_t addr = kbase + (ks >> 2) * (TK * 128) + sw128(kkey, chunk);
          uint32_t b0, b1, b2, b3;
          ldsm_x4(addr, b0, b1, b2, b3);
          mma_bf16_16816(acc[0], afrag[ks], b0, b1);
          mma_bf16_16816(acc[1], afrag[ks], b2, b3);
        }
        const int key_lo = t * TK + s16 * 16 + qc * 2;  // key of acc[0][0]
        // keys past the sequence take no part, whatever their rows hold
        float x[4], sv[4];
#pragma unroll
        for (int nn = 0; nn < 2; ++nn)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const bool in = key_lo + nn * 8 + e < kend;
            x[nn * 2 + e] = in ? acc[nn][e] * p.scale_log2 : -INFINITY;
            sv[nn * 2 + e] = in ? acc[nn][2 + e] : 0.f;
          }
        float tmax = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
        const float m_new = fmaxf(m_run, tmax);
        const float m_use = m_new == -INFINITY ? 0.f : m_new;
        const float alpha = ex2(m_run - m_use);
        float pr[4], ps[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) pr[e] = ex2(x[e] - m_use);
#pragma unroll
        for (int e = 0; e < 4; ++e) ps[e] = HAS_R ? pr[e] * sv[e] : 0.f;
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
          for (int jj = 0; jj < D / 8; ++jj) {
            o[jj][0] *= alpha; o[jj][1] *= alpha; o[jj][2] *= alpha; o[jj][3] *= alpha;
          }
        }
        if (t * TK + s16 * 16 + 16 <= kend)  // warp-uniform: all 16 keys live
          value_mma<D, TK>(o, pa, vbase, vkey, mi);
        else
          value_mma_masked<D, TK>(o, pa, vbase, vkey, mi, key_lo, kend);
      }
      // stage s is read: lane 0 refills it with the tile NS ahead in this warp's stream
      __syncwarp();
      if (lane == 0 && more) {
        issue(s);
        ++issued;
        more = ld.next(p, HN);
      }
    }
    if (!ok) break;

    // ---- this segment is finished in the warp: the row's l and c over the quad
    float l4 = l_run, c4 = c_run;
    l4 += __shfl_xor_sync(0xffffffffu, l4, 1);
    l4 += __shfl_xor_sync(0xffffffffu, l4, 2);
    c4 += __shfl_xor_sync(0xffffffffu, c4, 1);
    c4 += __shfl_xor_sync(0xffffffffu, c4, 2);
    if (gr < nh) {
      const size_t row = row0 + gr;
      if (p.rec_out) {
        float* rec = p.rec_out + row * (2 * D + 4);
        if (qc == 0) { rec[0] = m_run; rec[1] = l4; rec[2] = c4; rec[3] = 0.f; }
#pragma unroll
        for (int jj = 0; jj < D / 8; ++jj) {
          const int col = jj * 8 + qc * 2;
          *reinterpret_cast<float2*>(rec + 4 + col) = make_float2(o[jj][0], o[jj][1]);
          *reinterpret_cast<float2*>(rec + 4 + D + col) = make_float2(o[jj][2], o[jj][3]);
        }
      } else {
        const float inv = l4 > 0.f ? 1.f / l4 : 0.f;
        const float cl = c4 * inv;
#pragma unroll
        for (int jj = 0; jj < D / 8; ++jj) {
          const float a0 = o[jj][0] * inv, a1 = o[jj][1] * inv;
          const float r0 = a0 - (o[jj][2] * inv - cl * a0);
          const float r1 = a1 - (o[jj][3] * inv - cl * a1);
          *reinterpret_cast<__nv_bfloat162*>(p.out + row * D + jj * 8 + qc * 2) = __floats2bfloat162_rn(r0, r1);
        }
        if (qc == 0 && p.lse) p.lse[row] = l4 > 0.f ? (m_run + __log2f(l4)) * kLn2 : -INFINITY;
      }
    }
  }
  // every load issued must land before this CTA's shared memory goes away
  if (lane == 0)
    for (int j = max(k, issued - NS); j < issued; ++j)
      mbar_wait(smem_u32(&full[j % NS]), (j / NS) & 1, kErrDecodeDrain);
}

// Finishes what the split kernel left: the segments cut by a partition
// boundary (merging the partial states of the CTAs that shared each one),
// and the sequences with no live key (out = 0, lse = -inf).  A segment cut by
// boundaries is merged by the job of the split CTA that began it; this CTA
// takes the jobs of split CTAs blockIdx.x, blockIdx.x + gridDim.x, ...  It
// works out the same partition plan as the split kernel from the sequence
// lengths, before waiting for that grid, so that once the split grid is done
// only the partial states remain to be read.  Launched as a programmatic
// dependent of the split kernel; small enough (128 threads, ~4 KB of shared
// memory) to be resident beside two split CTAs on an SM.
template <int D>
__global__ void __launch_bounds__(kDecCombineThreads, 6)  // <= 85 registers: fits beside two split CTAs
plx_decode_combine_kernel(const DecodeParams p, int P) {
  constexpr int RF = DecodeCfg<D>::kRecFloats;
  constexpr int NT = kDecCombineThreads;
  constexpr int NW = NT / 32;
  constexpr int LANES = D / 4;  // lanes that hold a float4 of O1 and of O2
  constexpr int kMaxJobs = 4;
  __shared__ __align__(16) float s_mem[(NW * RF > 2 * NT + 4) ? NW * RF : 2 * NT + 4];
  __shared__ int4 s_job[kMaxJobs];  // {segment, first CTA, last CTA, first slot}
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // empty sequences: nothing of the split kernel touches their rows
  for (int b = blockIdx.x * NT + tid; b < p.B; b += gridDim.x * NT) {
    if (dec_live(p, b) != 0) continue;
    for (int h = 0; h < p.Hq; ++h) {
      const size_t row = static_cast<size_t>(b) * p.Hq + h;
      if (p.rec_out) {
        float* rec = p.rec_out + row * RF;
        rec[0] = -INFINITY; rec[1] = 0.f; rec[2] = 0.f; rec[3] = 0.f;
        for (int dd = 0; dd < 2 * D; ++dd) rec[4 + dd] = 0.f;
      } else {
        for (int dd = 0; dd < D; ++dd) p.out[row * D + dd] = __float2bfloat16(0.f);
        if (p.lse) p.lse[row] = -INFINITY;
      }
    }
  }

  // ---- the plan: which of this CTA's split CTAs began a segment it did not finish
  const int HN = p.Hkv * p.n_hgroups;
  int* scratch = reinterpret_cast<int*>(s_mem);
  dec_scan<NT>(p, scratch);
  const int T = scratch[2 * NT] * HN;
  const int tpc = dec_tpc(T, P);
  int njobs = 0;
  for (int c = blockIdx.x; c < P && njobs < kMaxJobs; c += gridDim.x) {
    const int t_begin = c * tpc;
    if (t_begin >= T) break;
    const int t_end = min(t_begin + tpc, T);
    dec_find<NT>(p, scratch, t_end - 1, HN);  // the segment of the range's last tile
    const int b = scratch[2 * NT + 1];
    const int nb = dec_ntiles(p, b);
    const int local = t_end - 1 - scratch[2 * NT + 2] * HN;
    const int j = local / nb, i = local % nb;
    const int seg_start = t_end - 1 - i;
    if (tid == 0 && i < nb - 1 && seg_start >= t_begin)
      s_job[njobs] = make_int4(b * HN + j, c, (seg_start + nb - 1) / tpc, seg_start == t_begin ? 2 * c : 2 * c + 1);
    njobs += (i < nb - 1 && seg_start >= t_begin) ? 1 : 0;
    __syncthreads();  // scratch is rewritten by the next dec_find
  }
  if (njobs == 0) return;  // uniform

  // wait until the split grid has completed and its writes are visible
  asm volatile("griddepcontrol.wait;" ::: "memory");
  float(*s_st)[RF] = reinterpret_cast<float(*)[RF]>(s_mem);
  for (int jb = 0; jb < njobs; ++jb) {
    const int4 job = s_job[jb];
    const int c0 = job.y, n = job.z - c0 + 1;
    const int b = job.x / HN, j = job.x % HN;
    const int g = j / p.n_hgroups, hg = j % p.n_hgroups;
    const int h0 = g * p.G + hg * 8, nh = min(8, p.G - hg * 8);
    // warps over (row, share of the partials): each row gets NW / nh warps,
    // or, with more rows than warps, each warp takes rows warp, warp + NW, ...
    const int wpr = nh >= NW ? 1 : NW / nh;
    for (int row0 = 0; row0 < nh; row0 += NW / wpr) {
      const int row = row0 + warp / wpr, sub = warp % wpr;
      if (row < nh && warp / wpr < NW / wpr) {
        float M = -INFINITY, L = 0.f, C = 0.f;
        float4 a1 = make_float4(0.f, 0.f, 0.f, 0.f), a2 = a1;
        const bool lv = lane < LANES;
        constexpr int R = kCombineDepth;
        for (int k0 = sub; k0 < n; k0 += R * wpr) {
          // R partials per round, all loaded before any is merged
          float4 h[R], x1[R], x2[R];
#pragma unroll
          for (int u = 0; u < R; ++u) {
            const int kk = k0 + u * wpr;
            h[u] = make_float4(-INFINITY, 0.f, 0.f, 0.f);
            x1[u] = x2[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (kk < n) {
              const int slot = kk == 0 ? job.w : 2 * (c0 + kk);
              const float* rec = p.ws + (static_cast<size_t>(slot) * p.rps + row) * RF;
              h[u] = __ldcg(reinterpret_cast<const float4*>(rec));
              if (lv) {
                x1[u] = __ldcg(reinterpret_cast<const float4*>(rec + 4) + lane);
                x2[u] = __ldcg(reinterpret_cast<const float4*>(rec + 4 + D) + lane);
              }
            }
          }
#pragma unroll
          for (int u = 0; u < R; ++u) {
            const float Mn = fmaxf(M, h[u].x);
            if (Mn == -INFINITY) continue;
            const float al = ex2(M - Mn), be = ex2(h[u].x - Mn);
            L = L * al + h[u].y * be;
            C = C * al + h[u].z * be;
            a1.x = a1.x * al + x1[u].x * be; a1.y = a1.y * al + x1[u].y * be;
            a1.z = a1.z * al + x1[u].z * be; a1.w = a1.w * al + x1[u].w * be;
            a2.x = a2.x * al + x2[u].x * be; a2.y = a2.y * al + x2[u].y * be;
            a2.z = a2.z * al + x2[u].z * be; a2.w = a2.w * al + x2[u].w * be;
            M = Mn;
          }
        }
        if (lane == 0) { s_st[warp][0] = M; s_st[warp][1] = L; s_st[warp][2] = C; }
        if (lv) {
          reinterpret_cast<float4*>(&s_st[warp][4])[lane] = a1;
          reinterpret_cast<float4*>(&s_st[warp][4 + D])[lane] = a2;
        }
      }
      __syncthreads();
      const int nrows = min(NW / wpr, nh - row0);
      for (int idx = tid; idx < nrows * D; idx += NT) {
        const int rr = idx / D, dd = idx % D;
        const int w0 = rr * wpr;
        float M = -INFINITY;
        for (int w = w0; w < w0 + wpr; ++w) M = fmaxf(M, s_st[w][0]);
        const float Mu = M == -INFINITY ? 0.f : M;
        float L = 0.f, C = 0.f, O1 = 0.f, O2 = 0.f;
        for (int w = w0; w < w0 + wpr; ++w) {
          const float be = ex2(s_st[w][0] - Mu);
          L += be * s_st[w][1];
          C += be * s_st[w][2];
          O1 += be * s_st[w][4 + dd];
          O2 += be * s_st[w][4 + D + dd];
        }
        const size_t orow = static_cast<size_t>(b) * p.Hq + h0 + row0 + rr;
        if (p.rec_out) {
          float* rec = p.rec_out + orow * RF;
          if (dd == 0) { rec[0] = M; rec[1] = L; rec[2] = C; rec[3] = 0.f; }
          rec[4 + dd] = O1;
          rec[4 + D + dd] = O2;
        } else {
          float res = 0.f;
          if (L > 0.f) {
            const float inv = 1.f / L;
            const float o1 = O1 * inv;
            res = o1 - (O2 * inv - (C * inv) * o1);
          }
          p.out[orow * D + dd] = __float2bfloat16(res);
          if (dd == 0 && p.lse) p.lse[orow] = L > 0.f ? (M + __log2f(L)) * kLn2 : -INFINITY;
        }
      }
      __syncthreads();
    }
  }
}

// Merges `blocks` state records per row into out and lse: record k of row r
// at recs + k * block_stride + r * row_stride floats (m in log2 units, l, c,
// pad, O1, O2).  The context-parallel merge of decode ranks or of prefill
// key chunks ([blocks, rows, 2D+4], block-major), and the merge of the parts
// of the chunked decode plan ([rows, parts, 2D+4]).  One
// warp per row at D = 128 (each lane holds four columns of O1 and of O2),
// two rows per warp at D = 64; every block's record is read once, coalesced.
template <int D>
__global__ void __launch_bounds__(256)
plx_record_merge_kernel(const float* __restrict__ recs, int blocks, long long rows, __nv_bfloat16* __restrict__ out,
                        float* __restrict__ lse, long long block_stride, long long row_stride) {
  constexpr int LPR = D / 4;  // lanes per row
  // launched as a programmatic dependent of the decode kernel (chunked plan):
  // wait until its records are written (a no-op otherwise)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const long long gl = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long row = gl / LPR;
  const int lane = static_cast<int>(gl % LPR);
  if (row >= rows) return;
  float M = -INFINITY, L = 0.f, C = 0.f;
  float4 a1 = make_float4(0.f, 0.f, 0.f, 0.f), a2 = a1;
  const size_t bstride = static_cast<size_t>(block_stride);
  int k = 0;
  for (; k < blocks; k += 2) {
    float4 h[2], x1[2], x2[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      h[u] = make_float4(-INFINITY, 0.f, 0.f, 0.f);
      x1[u] = x2[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (k + u < blocks) {
        const float* rec = recs + (k + u) * bstride + static_cast<size_t>(row) * row_stride;
        h[u] = __ldg(reinterpret_cast<const float4*>(rec));
        x1[u] = __ldcs(reinterpret_cast<const float4*>(rec + 4) + lane);
        x2[u] = __ldcs(reinterpret_cast<const float4*>(rec + 4 + D) + lane);
      }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const float Mn = fmaxf(M, h[u].x);
      if (Mn == -INFINITY) continue;
      const float al = ex2(M - Mn), be = ex2(h[u].x - Mn);
      L = L * al + h[u].y * be;
      C = C * al + h[u].z * be;
      a1.x = a1.x * al + x1[u].x * be; a1.y = a1.y * al + x1[u].y * be;
      a1.z = a1.z * al + x1[u].z * be; a1.w = a1.w * al + x1[u].w * be;
      a2.x = a2.x * al + x2[u].x * be; a2.y = a2.y * al + x2[u].y * be;
      a2.z = a2.z * al + x2[u].z * be; a2.w = a2.w * al + x2[u].w * be;
      M = Mn;
    }
  }
  float r[4] = {0.f, 0.f, 0.f, 0.f};
  if (L > 0.f) {
    const float inv = 1.f / L, cb = C * inv;
    const float o1[4] = {a1.x * inv, a1.y * inv, a1.z * inv, a1.w * inv};
    const float o2[4] = {a2.x * inv, a2.y * inv, a2.z * inv, a2.w * inv};
#pragma unroll
    for (int e = 0; e < 4; ++e) r[e] = o1[e] - (o2[e] - cb * o1[e]);
  }
  uint2 packed;
  packed.x = pack_bf16(r[0], r[1]);
  packed.y = pack_bf16(r[2], r[3]);
  *reinterpret_cast<uint2*>(out + static_cast<size_t>(row) * D + lane * 4) = packed;
  if (lane == 0 && lse) lse[row] = L > 0.f ? (M + __log2f(L)) * kLn2 : -INFINITY;
}

}  // namespace plx
