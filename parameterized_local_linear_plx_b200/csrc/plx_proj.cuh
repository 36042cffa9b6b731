// plx_proj.cuh -- the projection in front of the attention: q, k, v and the
// probe rho of every token from one GEMM, written straight into the layouts
// the attention kernels read.
//
// The pages make rho one more learned projection of the layer input, beside
// q, k and v (news.chathome.org, "Parallax: a parameterized local linear
// attention ...", section "What is Parallax"; gist.science, "Technical
// overview: Parallax ...", "Method: Parallax / Core mechanism": rho_i is
// parameterised).  So the four weights are stacked along the output
// dimension, W = [W_Q; W_K; W_V; W_R] ([Nout, d_model], rows = output
// features), and one GEMM y = x W^T (x [M, d_model], tokens as rows) yields
// all four.  The epilogue scatters each head's d columns of y to
//   - prefill: q, r [B, Hq, N, d] and k, v [B, Hkv, N, d] (token m = b N + t);
//   - decode (one token per sequence): q, r [B, Hq, d], and k, v straight into
//     the KV cache at row seqlens[b] of (b, kv head), contiguous or paged --
//     the append step of a decode, fused into the projection.
//
// Kernel.  Persistent CTAs (one per SM) walk 128 x BN output tiles (BN = 256;
// 64 for a decode step's few rows, so that more SMs share the weight stream).
// A TMA warp streams 64-wide K slices of x and W into a ring (128-byte
// swizzle); one thread issues tcgen05.mma (M = 128, N = BN, K = 16, bf16 in,
// fp32 accumulate) into one of two BN-column TMEM accumulators, so the next
// tile's MMAs run while four epilogue warps drain the previous one: TMEM ->
// registers -> bf16 -> a per-warp staging block in shared memory -> rows of
// the destination written with coalesced 16-byte stores.
#pragma once

#include "plx_ptx.cuh"
#include "plx_tcgen05.cuh"

namespace plx {

constexpr int kPjBM = 128, kPjBK = 64;
constexpr int kPjThreads = 192;                 // TMA warp, MMA warp, 4 epilogue warps
constexpr int kPjTmaWarp = 0, kPjMmaWarp = 1;
constexpr int kPjABytes = kPjBM * kPjBK * 2;    // 16 KB
constexpr int kPjEpiWarpBytes = 32 * 128 * 2;  // 32 rows x up to 128 columns, bf16

// Output tiles of 128 rows x BN columns: BN = 256 for prefill (many rows),
// BN = 64 for a decode step (few rows: more CTAs share the weight stream).
template <int BN>
struct ProjCfg {
  static constexpr int kBBytes = BN * kPjBK * 2;
  static constexpr int kStages = BN == 256 ? 4 : 8;
  static constexpr int kStageBytes = kPjABytes + kBBytes;
  static constexpr int kOffEpi = kStages * kStageBytes;
  static constexpr int kOffBar = kOffEpi + 4 * kPjEpiWarpBytes;
  static constexpr int kSmemBytes = kOffBar + 256 + 1024;  // barriers + alignment slack
  static constexpr uint32_t kTmemCols = 2 * BN;
};

// error codes of this kernel's bounded waits
constexpr unsigned kErrProjLoad = 0x401u, kErrProjMma = 0x402u, kErrProjEpi = 0x403u, kErrProjDrain = 0x404u;

struct ProjParams {
  int M, K, Nout, N, Hq, Hkv, d;   // M rows of x (tokens), K = d_model, N tokens per sequence
  int m_tiles, n_tiles, num_tiles, k_steps;
  __nv_bfloat16 *q, *k, *v, *r;    // destinations (r nullptr: W has no W_R rows; k, v unused in decode)
  int decode;                      // 1: row b is sequence b's new token; k, v go to the caches
  __nv_bfloat16 *kcache, *vcache;  // decode: [B, Hkv, S_max, d], or page pools [num_pages, Hkv, page_size, d]
  int S_max;
  const int32_t* seqlens;          // decode: slot of the new token
  int32_t* seqlens_out;            // decode: seqlens + 1 where the token was written (nullptr: not written)
  const int32_t* block_table;      // decode, paged caches: [B, max_pages] (nullptr: contiguous)
  int num_pages, page_size, page_shift, max_pages;
};

// 2-D tiled TMA load {c0 = column, c1 = row} into this CTA's shared memory.
__device__ __forceinline__ void tma_load_2d(const CUtensorMap* map, uint32_t dst, uint32_t bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}

// 32 lanes x 32 bits, 32 repetitions: thread t holds lane (base + t),
// columns c .. c+31 in registers 0..31.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

// Destination of row `m`, output columns col0 .. col0 + d - 1 (one head of one
// of q, k, v, r), or nullptr when nothing is written there.
__device__ __forceinline__ __nv_bfloat16* proj_dest(const ProjParams& p, int m, int col0) {
  const int d = p.d;
  const int nq = p.Hq * d, nkv = p.Hkv * d;
  int c = col0;
  if (c < nq) {
    const int b = m / p.N, t = m % p.N;
    return p.q + ((static_cast<size_t>(b) * p.Hq + c / d) * p.N + t) * d;
  }
  c -= nq;
  const bool is_k = c < nkv;
  if (c < 2 * nkv) {
    const int head = (is_k ? c : c - nkv) / d;
    if (!p.decode) {
      const int b = m / p.N, t = m % p.N;
      return (is_k ? p.k : p.v) + ((static_cast<size_t>(b) * p.Hkv + head) * p.N + t) * d;
    }
    const int slot = __ldg(p.seqlens + m);
    __nv_bfloat16* cache = is_k ? p.kcache : p.vcache;
    if (slot < 0) return nullptr;
    if (p.block_table == nullptr) {
      if (slot >= p.S_max) return nullptr;
      return cache + ((static_cast<size_t>(m) * p.Hkv + head) * p.S_max + slot) * d;
    }
    if (slot >= p.max_pages * p.page_size) return nullptr;
    const int pg = __ldg(p.block_table + static_cast<size_t>(m) * p.max_pages + (slot >> p.page_shift));
    if (pg < 0 || pg >= p.num_pages) return nullptr;
    return cache + ((static_cast<size_t>(pg) * p.Hkv + head) * p.page_size + (slot & (p.page_size - 1))) * d;
  }
  c -= 2 * nkv;
  if (p.r == nullptr) return nullptr;
  const int b = m / p.N, t = m % p.N;
  return p.r + ((static_cast<size_t>(b) * p.Hq + c / d) * p.N + t) * d;
}

template <int BN>
__global__ void __launch_bounds__(kPjThreads, 1)
plx_proj_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap wmap,
                const ProjParams p) {
  using Cfg = ProjCfg<BN>;
  constexpr int kPjStages = Cfg::kStages;
  constexpr int kPjBN = BN;
  constexpr int kPjStageBytes = Cfg::kStageBytes;
  constexpr uint32_t kPjTmemCols = Cfg::kTmemCols;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::kOffBar);
  uint64_t* empty = full + kPjStages;
  uint64_t* acc_full = empty + kPjStages;  // [2]
  uint64_t* acc_empty = acc_full + 2;      // [2]
  uint64_t* fin = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPjStages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&acc_full[b]), 1);
      mbar_init(smem_u32(&acc_empty[b]), 4);  // one arrival per epilogue warp
    }
    mbar_init(smem_u32(fin), 1);
    fence_barrier_init();
  }
  if (warp == kPjMmaWarp) {
    tc::tmem_alloc(smem_u32(tmem_slot), kPjTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == kPjTmaWarp) {
    // ================================================================ loads
    if (lane == 0) {
      tma_prefetch_desc(&xmap);
      tma_prefetch_desc(&wmap);
      int it = 0;
      for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
        const int m0 = (tile / p.n_tiles) * kPjBM, n0 = (tile % p.n_tiles) * kPjBN;
        bool ok = true;
        for (int kb = 0; kb < p.k_steps; ++kb, ++it) {
          const int s = it % kPjStages;
          if (it >= kPjStages && !mbar_wait(smem_u32(&empty[s]), ((it / kPjStages) - 1) & 1, kErrProjLoad)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&full[s]);
          mbar_arrive_expect_tx(fb, kPjStageBytes);
          const uint32_t a = smem_u32(smem + s * kPjStageBytes);
          tma_load_2d(&xmap, a, fb, kb * kPjBK, m0);
          tma_load_2d(&wmap, a + kPjABytes, fb, kb * kPjBK, n0);
        }
        if (!ok) break;
      }
      // every load issued lands before the CTA's shared memory goes away
      for (int j = max(0, it - kPjStages); j < it; ++j)
        mbar_wait(smem_u32(&full[j % kPjStages]), (j / kPjStages) & 1, kErrProjDrain);
    }
  } else if (warp == kPjMmaWarp) {
    // ================================================================ MMA issue
    if (lane == 0) {
      constexpr uint32_t idesc = tc::idesc_bf16_f32(kPjBM, kPjBN, 0, 0);  // x and W both K-major
      const uint64_t da = tc::smem_desc_sw128(smem_u32(smem), 16, 1024);
      const uint64_t db = tc::smem_desc_sw128(smem_u32(smem + kPjABytes), 16, 1024);
      constexpr uint64_t kStep = kPjStageBytes >> 4;  // descriptor units
      int it = 0, lt = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x, ++lt) {
        const int buf = lt & 1;
        if (lt >= 2 && !mbar_wait(smem_u32(&acc_empty[buf]), ((lt >> 1) - 1) & 1, kErrProjMma)) break;
        tc::fence_after_sync();
        const uint32_t dst = tmem + buf * kPjBN;
        for (int kb = 0; kb < p.k_steps; ++kb, ++it) {
          const int s = it % kPjStages;
          if (!mbar_wait(smem_u32(&full[s]), (it / kPjStages) & 1, kErrProjMma)) { ok = false; break; }
          tc::fence_after_sync();
#pragma unroll
          for (int ks = 0; ks < kPjBK / 16; ++ks)
            tc::mma_ss(dst, da + s * kStep + ks * 2, db + s * kStep + ks * 2, idesc, (kb | ks) ? 1u : 0u);
          tc::commit(smem_u32(&empty[s]));
        }
        if (ok) tc::commit(smem_u32(&acc_full[buf]));
      }
      // every MMA issued completes before tensor memory is freed
      tc::commit(smem_u32(fin));
      mbar_wait(smem_u32(fin), 0, kErrProjMma);
    }
  } else {
    // ================================================================ epilogue
    const int quad = warp & 3;  // the TMEM lane quarter this warp may read
    uint8_t* stg = smem + Cfg::kOffEpi + quad * kPjEpiWarpBytes;
    const int d = p.d;
    const int cw = d < kPjBN ? d : kPjBN;  // columns per destination chunk (within one head)
    const int cpr = cw / 8;                // 16-byte chunks per destination row
    int lt = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++lt) {
      const int buf = lt & 1;
      const bool got = mbar_wait(smem_u32(&acc_full[buf]), (lt >> 1) & 1, kErrProjEpi);
      if (!__all_sync(0xffffffffu, got)) break;
      tc::fence_after_sync();
      const int m0 = (tile / p.n_tiles) * kPjBM, n0 = (tile % p.n_tiles) * kPjBN;
      const int rbase = m0 + quad * 32;  // this warp's first row
      for (int c0 = 0; c0 < kPjBN && n0 + c0 < p.Nout; c0 += cw) {
        // TMEM columns c0 .. c0 + cw - 1 of this warp's 32 rows -> bf16 staging
        for (int sub = 0; sub < cw / 32; ++sub) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(quad * 32) << 16) + buf * kPjBN + c0 + sub * 32, v);
          tc::wait_ld();
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            uint4 w4;
            w4.x = pack_bf16(__uint_as_float(v[8 * ch + 0]), __uint_as_float(v[8 * ch + 1]));
            w4.y = pack_bf16(__uint_as_float(v[8 * ch + 2]), __uint_as_float(v[8 * ch + 3]));
            w4.z = pack_bf16(__uint_as_float(v[8 * ch + 4]), __uint_as_float(v[8 * ch + 5]));
            w4.w = pack_bf16(__uint_as_float(v[8 * ch + 6]), __uint_as_float(v[8 * ch + 7]));
            const int chunk = (sub * 4 + ch) ^ (lane & (cpr - 1));
            *reinterpret_cast<uint4*>(stg + lane * (cw * 2) + chunk * 16) = w4;
          }
        }
        __syncwarp();
        // each lane finds the destination of its own row once (the index
        // arithmetic has runtime divisors); the warp then writes its 32 rows,
        // cpr lanes per row, 16 bytes each, taking row pointers by shuffle
        const int col = n0 + c0, in_head = col & (d - 1);
        const int m_me = rbase + lane;
        __nv_bfloat16* mine = m_me < p.M ? proj_dest(p, m_me, col - in_head) : nullptr;
        const unsigned long long my_dst =
            mine ? reinterpret_cast<unsigned long long>(mine + in_head) : 0ull;
        const int rshift = __ffs(cpr) - 1;  // cpr is a power of two
        for (int idx = lane; idx < 32 * cpr; idx += 32) {
          const int rr = idx >> rshift, ch = idx & (cpr - 1);
          const unsigned long long dst = __shfl_sync(0xffffffffu, my_dst, rr);
          if (dst == 0ull) continue;
          const uint4 w4 = *reinterpret_cast<const uint4*>(stg + rr * (cw * 2) + ((ch ^ (rr & (cpr - 1))) * 16));
          *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(dst) + ch * 8) = w4;
        }
        __syncwarp();
      }
      if (p.decode && p.seqlens_out && n0 == 0) {
        // the new token is in the cache: one thread per sequence advances its length
        const int m = rbase + lane;
        if (m < p.M) {
          const int slot = __ldg(p.seqlens + m);
          const int cap = p.block_table ? p.max_pages * p.page_size : p.S_max;
          bool written = slot >= 0 && slot < cap;
          if (written && p.block_table) {
            const int pg = __ldg(p.block_table + static_cast<size_t>(m) * p.max_pages + (slot >> p.page_shift));
            written = pg >= 0 && pg < p.num_pages;
          }
          p.seqlens_out[m] = written ? slot + 1 : slot;
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&acc_empty[buf]));
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == kPjMmaWarp) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kPjTmemCols);
  }
}

}  // namespace plx
