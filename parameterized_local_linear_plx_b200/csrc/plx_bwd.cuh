// plx_bwd.cuh -- gradients of the Parallax attention forward on sm_100a.
//
// The forward is that of gist.science, "Technical overview: Parallax -
// parameterized local linear attention for language modeling", section
// "Method: Parallax / Core mechanism" (o = o_SA - Sigma_KV rho, eta = 0), in
// its effective-weight form o_i = sum_j w_hat_ij v_j with
// w_hat_ij = w_ij (1 - s_ij + s_bar_i), s_ij = rho_i . k_j.  The pages give no
// backward; the gradient of the loss sum_i dO_i . o_i is
//
//   g_ij  = dO_i . v_j,   g_bar_i = dO_i . o_bar_i,   Dd_i = dO_i . o_i + s_bar_i g_bar_i
//   dV_j  = sum_i w_hat_ij dO_i
//   dS_ij = w_ij (g_bar_i - g_ij)
//   dA_ij = w_ij (g_ij (1 - s_ij + s_bar_i) + s_ij g_bar_i - Dd_i)
//   dQ_i  = scale sum_j dA_ij k_j,   dR_i = sum_j dS_ij k_j
//   dK_j  = sum_i (scale dA_ij) q_i + dS_ij rho_i
//
// with w_ij = exp(scale q_i . k_j - lse_i) recomputed from the forward's lse,
// and o_bar, s_bar kept by the training forward.
//
// Kernels:
//   * plx_bwd_pre_kernel: one warp per query row: g_bar and Dd.
//   * plx_bwd_q_kernel (dQ, dR): one CTA per 64-query tile, with the stacked
//     [Q;R] operand of the forward (rows 32w..32w+15: queries 16w..16w+15; rows
//     32w+16..32w+31: their probes).  Per 128-key tile: S = [Q;R] K^T and
//     G = [dO;0] V^T (dO in the query slots of a second stacked operand and
//     zeros in the probe slots, so g lands in the query lanes beside a), then
//     the element-wise warps write [scale dA ; dS] in bf16 over S and one MMA
//     [scale dA ; dS] K accumulates [dQ ; dR] in tensor memory.  S has two
//     buffers: the scores of tile j+1 are computed during the element-wise
//     pass of tile j, and only G(j+1) stands between two passes.
//   * plx_bwd_kv_kernel (dK, dV): one CTA per 128-key tile, keys as the MMA
//     rows.  For each 64-query tile of each query head of the KV group:
//     [A^T | S^T] = K [Q;R]^T and G^T = V dO^T; per (key, query) the
//     element-wise warps write W_hat^T, scale dA^T and dS^T in bf16; then
//     dV += W_hat^T dO and dK += [scale dA^T | dS^T] [Q;R] (the stacked tile is
//     the K-major B of the first product and the MN-major B of the last).
//     G^T has two buffers in tensor memory, so the next tile's G^T and this
//     tile's dV products run during the element-wise pass; only dK and the
//     next scores stand between two passes.  Each CTA owns its output rows:
//     no atomics anywhere.
//   * In both: warps 0-15 element-wise.  Warp w reads TMEM lanes
//     32(w%4)..32(w%4)+31 and one quarter (w/4) of the columns; every
//     (key, query) element is independent, so the warps share nothing, and
//     each writes its bf16 results over fp32 columns it has itself already
//     read.  Warp 16 issues the TMA loads, warp 17 allocates tensor memory and
//     one of its threads issues every MMA.  Every wait is bounded (device
//     error word).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include <cstdint>

#include "plx_ptx.cuh"
#include "plx_tcgen05.cuh"

namespace plx {

constexpr int kBwdBM = 64;        // queries per tile (128 stacked rows with their probes)
constexpr int kBwdBN = 128;       // keys per tile
constexpr int kBwdElemWarps = 16;
constexpr int kBwdThreads = 32 * (kBwdElemWarps + 2);  // element-wise warps, TMA warp, MMA warp
constexpr int kBwdTmaWarp = kBwdElemWarps;
constexpr int kBwdMmaWarp = kBwdElemWarps + 1;
constexpr int kBwdStages = 3;

struct BwdParams {
  __nv_bfloat16* dq;  // [B, Hq, N, D]
  __nv_bfloat16* dr;  // [B, Hq, N, D] or nullptr
  __nv_bfloat16* dk;  // [B, Hkv, N, D]
  __nv_bfloat16* dv;  // [B, Hkv, N, D]
  const float* lse;   // [B, Hq, N]
  const float* gbar;  // [B, Hq, N]  dO . o_bar
  const float* dd;    // [B, Hq, N]  dO . o + s_bar g_bar
  const float* sbar;  // [B, Hq, N] or nullptr (rho = 0)
  int B, Hq, Hkv, N, G;
  int n_qtiles;  // ceil(N / 64)
  int n_ktiles;  // ceil(N / 128)
  int causal;
  float scale, scale_log2;
};

// ---------------------------------------------------------------- preprocess
// g_bar = dO . o_bar and Dd = dO . o + s_bar g_bar for every query row (one
// warp per row; lane l reads the 32-bit words l, l + 32, ... of the row).
template <int D>
__global__ void __launch_bounds__(256) plx_bwd_pre_kernel(const __nv_bfloat16* __restrict__ dout,
                                                          const __nv_bfloat16* __restrict__ out,
                                                          const __nv_bfloat16* __restrict__ obar,
                                                          const float* __restrict__ sbar, float* __restrict__ gbar,
                                                          float* __restrict__ dd, long long rows) {
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const uint32_t* pd = reinterpret_cast<const uint32_t*>(dout + row * D);
  const uint32_t* po = reinterpret_cast<const uint32_t*>(out + row * D);
  const uint32_t* pb = reinterpret_cast<const uint32_t*>(obar + row * D);
  float go = 0.f, gb = 0.f;
#pragma unroll
  for (int i = 0; i < D / 64; ++i) {
    const uint32_t a = __ldg(pd + 32 * i + lane), o = __ldg(po + 32 * i + lane), b = __ldg(pb + 32 * i + lane);
    go = fmaf(bf16_lo(a), bf16_lo(o), go);
    go = fmaf(bf16_hi(a), bf16_hi(o), go);
    gb = fmaf(bf16_lo(a), bf16_lo(b), gb);
    gb = fmaf(bf16_hi(a), bf16_hi(b), gb);
  }
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) {
    go += __shfl_xor_sync(0xffffffffu, go, m);
    gb += __shfl_xor_sync(0xffffffffu, gb, m);
  }
  if (lane == 0) {
    const float sb = sbar ? sbar[row] : 0.f;
    gbar[row] = gb;
    dd[row] = go + sb * gb;
  }
}

// ---------------------------------------------------------------- dQ, dR
// Keys come in tiles of 128 (N = 128 score MMAs: half the instructions per key
// of 64-key tiles).  Tensor memory holds two score buffers, one G buffer and
// [dQ ; dR]: the scores of tile j+1 run during the element-wise pass of tile
// j, and only G(j+1) (512 tensor cycles) stands between two passes; [dQ ; dR]
// of tile j and the scores of j+2 follow it in the tensor pipe.  K and V have
// rings of their own: V is free once G has read it, K only after the
// [dQ ; dR] product.
constexpr int kBwdQBN = 128;     // keys per tile of the query-side kernel
constexpr int kBwdQKStages = 3;  // K ring
constexpr int kBwdQVStages = 2;  // V ring

template <int D>
struct BwdQCfg {
  static constexpr int kCB = D / 64;              // 128-byte column blocks per row
  static constexpr int kBlock = 128 * 128;        // one [128 rows x 128 B] block
  static constexpr int kKVBlock = kBwdQBN * 128;  // one [128 keys x 128 B] block
  static constexpr int kTileBytes = kCB * kBlock;  // a 128-row stacked tile
  static constexpr int kKVBytes = kCB * kKVBlock;  // a 128-key K or V tile
  static constexpr int kOffQR = 0;
  static constexpr int kOffDO = kTileBytes;        // [dO ; 0] stacked like [Q ; R]
  static constexpr int kOffK = 2 * kTileBytes;
  static constexpr int kOffV = kOffK + kBwdQKStages * kKVBytes;
  static constexpr int kOffBar = kOffV + kBwdQVStages * kKVBytes;
  static constexpr int kSmemBytes = kOffBar + 256 + 1024;
  // tensor memory: S of tile j at 128 (j & 1), G at 256, [dQ ; dR] at 384
  static constexpr uint32_t kColS = 0, kColG = 256, kColAcc = 384, kTmemCols = 512;
};

template <int D, bool HAS_R>
__global__ void __launch_bounds__(kBwdThreads, 1)
plx_bwd_q_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap rmap,
                 const __grid_constant__ CUtensorMap omap, const __grid_constant__ CUtensorMap kmap,
                 const __grid_constant__ CUtensorMap vmap, const BwdParams p) {
  using Cfg = BwdQCfg<D>;
  constexpr int NK = kBwdQKStages, NV = kBwdQVStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kOffBar);
  uint64_t* q_full = bars;              // [1] [Q;R] and [dO;0] landed
  uint64_t* k_full = bars + 1;          // [NK]
  uint64_t* k_empty = k_full + NK;      // [NK]
  uint64_t* v_full = k_empty + NK;      // [NV]
  uint64_t* v_empty = v_full + NV;      // [NV]
  uint64_t* s_full = v_empty + NV;      // [2] S of a key tile in TMEM buffer j & 1
  uint64_t* g_full = s_full + 2;        // [1] G of a key tile in TMEM
  uint64_t* p_ready = g_full + 1;       // [1] [dA ; dS] written (one arrival per element-wise warp)
  uint64_t* o_done = p_ready + 1;       // [1] every MMA complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_done + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int per = p.B * p.Hq;
  const int qt = p.n_qtiles - 1 - static_cast<int>(blockIdx.x) / per;  // longest causal rows first
  const int bh = static_cast<int>(blockIdx.x) % per;                   // b * Hq + h
  const int b = bh / p.Hq, h = bh % p.Hq;
  const int q0 = qt * kBwdBM;
  const int plane_kv = b * p.Hkv + h / p.G;
  const int qmax = min(p.N - 1, q0 + kBwdBM - 1);
  const int n_all = (p.N + kBwdQBN - 1) / kBwdQBN;
  const int nkv = p.causal ? qmax / kBwdQBN + 1 : n_all;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(q_full), 1);
    for (int s = 0; s < NK; ++s) {
      mbar_init(smem_u32(&k_full[s]), 1);
      mbar_init(smem_u32(&k_empty[s]), 1);
    }
    for (int s = 0; s < NV; ++s) {
      mbar_init(smem_u32(&v_full[s]), 1);
      mbar_init(smem_u32(&v_empty[s]), 1);
    }
    mbar_init(smem_u32(&s_full[0]), 1);
    mbar_init(smem_u32(&s_full[1]), 1);
    mbar_init(smem_u32(g_full), 1);
    mbar_init(smem_u32(p_ready), kBwdElemWarps);  // one arrival per element-wise warp
    mbar_init(smem_u32(o_done), 1);
    fence_barrier_init();
  }
  {
    // zero the probe slots of [dO ; 0] (and of [Q ; R] when rho = 0): TMA writes only the other rows
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    const int n_tiles = HAS_R ? 1 : 2;
    for (int i = threadIdx.x; i < n_tiles * Cfg::kCB * 4 * 16 * 8; i += kBwdThreads) {
      const int c16 = i & 7, row = (i >> 3) & 15, w = (i >> 7) & 3, cb = (i >> 9) % Cfg::kCB,
                t = (i >> 9) / Cfg::kCB;
      const int base = (HAS_R || t == 1) ? Cfg::kOffDO : Cfg::kOffQR;
      uint8_t* dst = smem + base + cb * Cfg::kBlock + (32 * w + 16 + row) * 128 + c16 * 16;
      *reinterpret_cast<uint4*>(dst) = z;
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == kBwdMmaWarp) {
    tc::tmem_alloc(smem_u32(tmem_slot), Cfg::kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;

  if (warp == kBwdTmaWarp) {
    // ================================================================ TMA producer
    if (lane == 0) {
      const int plane = bh;
      {
        const uint32_t fb = smem_u32(q_full);
        mbar_arrive_expect_tx(fb, (HAS_R ? 3 : 2) * Cfg::kTileBytes / 2);
#pragma unroll
        for (int wq = 0; wq < 4; ++wq)
#pragma unroll
          for (int cb = 0; cb < Cfg::kCB; ++cb) {
            const uint32_t off = cb * Cfg::kBlock + (32 * wq) * 128;
            tma_load_3d(&qmap, smem_u32(smem + Cfg::kOffQR + off), fb, cb * 64, q0 + 16 * wq, plane);
            if (HAS_R) tma_load_3d(&rmap, smem_u32(smem + Cfg::kOffQR + off + 16 * 128), fb, cb * 64, q0 + 16 * wq, plane);
            tma_load_3d(&omap, smem_u32(smem + Cfg::kOffDO + off), fb, cb * 64, q0 + 16 * wq, plane);
          }
      }
      int issued_k = 0, issued_v = 0;
      for (int j = 0; j < nkv; ++j) {
        const int sk = j % NK, sv = j % NV;
        if (j >= NK && !mbar_wait_sleep(smem_u32(&k_empty[sk]), ((j / NK) - 1) & 1, kErrBwdLoad)) { ok = false; break; }
        {
          const uint32_t fb = smem_u32(&k_full[sk]);
          mbar_arrive_expect_tx(fb, Cfg::kKVBytes);
#pragma unroll
          for (int cb = 0; cb < Cfg::kCB; ++cb)
            tma_load_3d(&kmap, smem_u32(smem + Cfg::kOffK + sk * Cfg::kKVBytes + cb * Cfg::kKVBlock), fb, cb * 64,
                        j * kBwdQBN, plane_kv);
          issued_k = j + 1;
        }
        if (j >= NV && !mbar_wait_sleep(smem_u32(&v_empty[sv]), ((j / NV) - 1) & 1, kErrBwdLoad)) { ok = false; break; }
        {
          const uint32_t fb = smem_u32(&v_full[sv]);
          mbar_arrive_expect_tx(fb, Cfg::kKVBytes);
#pragma unroll
          for (int cb = 0; cb < Cfg::kCB; ++cb)
            tma_load_3d(&vmap, smem_u32(smem + Cfg::kOffV + sv * Cfg::kKVBytes + cb * Cfg::kKVBlock), fb, cb * 64,
                        j * kBwdQBN, plane_kv);
          issued_v = j + 1;
        }
      }
      if (!ok) {  // let every issued load land before the CTA can exit
        mbar_wait(smem_u32(q_full), 0, kErrBwdDrain);
        for (int j = max(0, issued_k - NK); j < issued_k; ++j) mbar_wait(smem_u32(&k_full[j % NK]), (j / NK) & 1, kErrBwdDrain);
        for (int j = max(0, issued_v - NV); j < issued_v; ++j) mbar_wait(smem_u32(&v_full[j % NV]), (j / NV) & 1, kErrBwdDrain);
      }
    }
  } else if (warp == kBwdMmaWarp) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = tc::idesc_bf16_f32(128, kBwdQBN, 0, 0);  // [X;Y] x Z^T, both K-major
      constexpr uint32_t idesc_o = tc::idesc_bf16_f32(128, D, 0, 1);        // [dA;dS] x K, K MN-major
      constexpr uint64_t kStageStep = Cfg::kKVBytes >> 4;
      const uint64_t d_qr = tc::smem_desc_sw128(smem_u32(smem + Cfg::kOffQR), 16, 1024);
      const uint64_t d_do = tc::smem_desc_sw128(smem_u32(smem + Cfg::kOffDO), 16, 1024);
      const uint64_t d_k = tc::smem_desc_sw128(smem_u32(smem + Cfg::kOffK), 16, 1024);
      const uint64_t d_v = tc::smem_desc_sw128(smem_u32(smem + Cfg::kOffV), 16, 1024);
      const uint64_t d_kmn = tc::smem_desc_sw128(smem_u32(smem + Cfg::kOffK), Cfg::kKVBlock, 1024);
      // Per key tile j, in issue order (the tensor pipe runs them in that
      // order): after the element-wise pass of j, G(j+1) (the pass of j+1 then
      // waits only for it: its scores were computed during the pass of j),
      // [dQ ; dR] += [scale dA ; dS] K (the last reader of S buffer j & 1),
      // then the scores of j+2 into that buffer.
      auto issue_s = [&](int j) -> bool {
        const int s = j % NK;
        if (!mbar_wait(smem_u32(&k_full[s]), (j / NK) & 1, kErrBwdMma)) return false;
        tc::fence_after_sync();
        const uint32_t cs = tmem + Cfg::kColS + 128 * static_cast<uint32_t>(j & 1);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint64_t koff_a = static_cast<uint64_t>(((ks >> 2) * Cfg::kBlock + (ks & 3) * 32) >> 4);
          const uint64_t koff_b = static_cast<uint64_t>(((ks >> 2) * Cfg::kKVBlock + (ks & 3) * 32) >> 4);
          tc::mma_ss(cs, d_qr + koff_a, d_k + s * kStageStep + koff_b, idesc_s, ks > 0 ? 1u : 0u);
        }
        tc::commit(smem_u32(&s_full[j & 1]));
        return true;
      };
      auto issue_g = [&](int j) -> bool {
        const int s = j % NV;
        if (!mbar_wait(smem_u32(&v_full[s]), (j / NV) & 1, kErrBwdMma)) return false;
        tc::fence_after_sync();
        const uint32_t cg = tmem + Cfg::kColG;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint64_t koff_a = static_cast<uint64_t>(((ks >> 2) * Cfg::kBlock + (ks & 3) * 32) >> 4);
          const uint64_t koff_b = static_cast<uint64_t>(((ks >> 2) * Cfg::kKVBlock + (ks & 3) * 32) >> 4);
          tc::mma_ss(cg, d_do + koff_a, d_v + s * kStageStep + koff_b, idesc_s, ks > 0 ? 1u : 0u);
        }
        tc::commit(smem_u32(&v_empty[s]));  // G is V's only reader
        tc::commit(smem_u32(g_full));
        return true;
      };
      ok = mbar_wait(smem_u32(q_full), 0, kErrBwdMma);
      if (ok && nkv > 0) ok = issue_g(0) && issue_s(0) && (nkv < 2 || issue_s(1));
      for (int j = 0; j < nkv && ok; ++j) {
        // the element-wise pass of j is over: G and S buffer j & 1 may be reused
        if (!mbar_wait(smem_u32(p_ready), j & 1, kErrBwdMma)) { ok = false; break; }
        tc::fence_after_sync();
        if (j + 1 < nkv && !issue_g(j + 1)) { ok = false; break; }
        // A = the bf16 pairs of keys 16kk..16kk+15: warp part c wrote keys
        // 32c..32c+31 as pairs at columns 32c..32c+15 of its S buffer
        const int sk = j % NK;
        const uint32_t cs = tmem + Cfg::kColS + 128 * static_cast<uint32_t>(j & 1);
#pragma unroll
        for (int kk = 0; kk < kBwdQBN / 16; ++kk)
          tc::mma_ts(tmem + Cfg::kColAcc, cs + 32 * (kk >> 1) + 8 * (kk & 1),
                     d_kmn + sk * kStageStep + static_cast<uint64_t>((kk * 2048) >> 4), idesc_o,
                     (j > 0 || kk > 0) ? 1u : 0u);
        tc::commit(smem_u32(&k_empty[sk]));
        if (j + 2 < nkv && !issue_s(j + 2)) { ok = false; break; }
      }
      tc::commit(smem_u32(o_done));  // also on abort: every issued MMA completes before dealloc
      mbar_wait(smem_u32(o_done), 0, kErrBwdMma);
    }
  } else {
    // ================================================================ element-wise + epilogue
    // warp (wq, part): rows of TMEM quadrant wq, keys 32part..32part+31 of each tile
    const int wq = warp & 3, part = warp >> 2;
    const int c4 = lane & 3;
    const int r_lo = lane >> 2;
    const uint32_t lane_a = static_cast<uint32_t>(32 * wq) << 16;
    const uint32_t lane_s = static_cast<uint32_t>(32 * wq + 16) << 16;
    const int q_lo = q0 + 16 * wq + r_lo, q_hi = q_lo + 8;
    const size_t rb = static_cast<size_t>(bh) * p.N;
    // per-row statistics (rows past N: lse = +inf gives w = 0)
    float l2_lo = INFINITY, l2_hi = INFINITY, sb_lo = 0.f, sb_hi = 0.f, gb_lo = 0.f, gb_hi = 0.f, dd_lo = 0.f,
          dd_hi = 0.f;
    if (q_lo < p.N) {
      l2_lo = p.lse[rb + q_lo] * kLog2e;
      gb_lo = p.gbar[rb + q_lo];
      dd_lo = p.dd[rb + q_lo];
      if (HAS_R) sb_lo = p.sbar[rb + q_lo];
    }
    if (q_hi < p.N) {
      l2_hi = p.lse[rb + q_hi] * kLog2e;
      gb_hi = p.gbar[rb + q_hi];
      dd_hi = p.dd[rb + q_hi];
      if (HAS_R) sb_hi = p.sbar[rb + q_hi];
    }
    // the per-row constants as packed pairs (both elements of a pair share the row):
    // -lse log2(e), 1 + s_bar, g_bar, -Dd
    const uint64_t nl_lo = f2(-l2_lo, -l2_lo), nl_hi = f2(-l2_hi, -l2_hi);
    const uint64_t f_lo = f2(1.f + sb_lo, 1.f + sb_lo), f_hi = f2(1.f + sb_hi, 1.f + sb_hi);
    const uint64_t gb2_lo = f2(gb_lo, gb_lo), gb2_hi = f2(gb_hi, gb_hi);
    const uint64_t nd_lo = f2(-dd_lo, -dd_lo), nd_hi = f2(-dd_hi, -dd_hi);
    const uint64_t c_sl2 = f2(p.scale_log2, p.scale_log2), c_m1 = f2(-1.f, -1.f), c_sc = f2(p.scale, p.scale);
    for (int j = 0; j < nkv; ++j) {
      const bool landed = mbar_wait_sleep(smem_u32(&s_full[j & 1]), (j >> 1) & 1, kErrBwdElem) &&
                          mbar_wait_sleep(smem_u32(g_full), j & 1, kErrBwdElem);
      if (!__all_sync(0xffffffffu, landed)) { ok = false; break; }
      tc::fence_after_sync();
      const uint32_t cs = Cfg::kColS + 128 * static_cast<uint32_t>(j & 1) + 32 * part;
      const uint32_t ta = tmem + lane_a + cs, ts = tmem + lane_s + cs;
      const uint32_t tg = tmem + lane_a + Cfg::kColG + 32 * part;
      uint32_t ra[16], rs[16], rg[16];
      tc::ld_16x256b_x4(ta, ra);
      tc::ld_16x256b_x4(ts, rs);
      tc::ld_16x256b_x4(tg, rg);
      tc::wait_ld();
      // masks only where some (query, key) of this warp is out of the set:
      // keys past N, or (causal) a key of the warp after its first row
      const int kw = j * kBwdQBN + 32 * part;  // this warp's first key
      const bool need_mask = (kw + 31 >= p.N) || (p.causal && kw + 31 > q0 + 16 * wq);
      // register i: rep gg = i/4, e = i%4; key = 128j + 32part + 8gg + 2c4 + (e&1);
      // row lo for e < 2, row hi for e >= 2.  Registers (4gg, 4gg+1) and
      // (4gg+2, 4gg+3) are key pairs of one row: packed f32x2 arithmetic.
      uint32_t pa[8], pd[8];
#pragma unroll
      for (int h2 = 0; h2 < 8; ++h2) {
        const int i = 2 * h2;
        const bool hi = (h2 & 1) != 0;
        const uint64_t A = f2(__uint_as_float(ra[i]), __uint_as_float(ra[i + 1]));
        const uint64_t S = f2(__uint_as_float(rs[i]), __uint_as_float(rs[i + 1]));
        const uint64_t G = f2(__uint_as_float(rg[i]), __uint_as_float(rg[i + 1]));
        const uint64_t X = f2_fma(A, c_sl2, hi ? nl_hi : nl_lo);
        float w0 = ex2(f2_lo(X)), w1 = ex2(f2_hi(X));
        if (need_mask) {
          const int key = kw + 8 * (h2 >> 1) + 2 * c4;
          const int q = hi ? q_hi : q_lo;
          if (key >= p.N || (p.causal && key > q)) w0 = 0.f;
          if (key + 1 >= p.N || (p.causal && key + 1 > q)) w1 = 0.f;
        }
        const uint64_t W = f2(w0, w1);
        const uint64_t Gb = hi ? gb2_hi : gb2_lo;
        const uint64_t F = f2_fma(S, c_m1, hi ? f_hi : f_lo);                  // 1 + s_bar - s
        const uint64_t DS = f2_mul(W, f2_fma(G, c_m1, Gb));                     // w (g_bar - g)
        const uint64_t U = f2_fma(G, F, f2_fma(S, Gb, hi ? nd_hi : nd_lo));    // g f + s g_bar - Dd
        const uint64_t DA = f2_mul(f2_mul(W, c_sc), U);
        pa[h2] = pack_bf16(f2_lo(DA), f2_hi(DA));
        pd[h2] = pack_bf16(f2_lo(DS), f2_hi(DS));
      }
      // bf16 pairs over the first 16 of this warp's own 32 fp32 columns
      tc::st_16x128b_x4(ta, pa);
      tc::st_16x128b_x4(ts, pd);
      tc::wait_st();
      tc::fence_before_sync();
      __syncwarp();  // every lane's stores are complete: one lane arrives for the warp
      if (lane == 0) mbar_arrive(smem_u32(p_ready));
    }
    if (ok) {
      const bool done = mbar_wait_sleep(smem_u32(o_done), 0, kErrBwdElem);
      if (__all_sync(0xffffffffu, done)) {
        tc::fence_after_sync();
        // this warp's quarter of the columns: [part * D/4, (part + 1) * D/4)
        const uint32_t t1 = tmem + lane_a + Cfg::kColAcc, t2 = tmem + lane_s + Cfg::kColAcc;
#pragma unroll
        for (int ch = 0; ch < D / 64; ++ch) {
          const int cbase = part * (D / 4) + 16 * ch;
          uint32_t o1[8], o2[8];
          tc::ld_16x256b_x2(t1 + cbase, o1);
          tc::ld_16x256b_x2(t2 + cbase, o2);
          tc::wait_ld();
#pragma unroll
          for (int gg = 0; gg < 2; ++gg) {
            const int col = cbase + 8 * gg + 2 * c4;
            if (q_lo < p.N) {
              *reinterpret_cast<uint32_t*>(p.dq + (rb + q_lo) * D + col) =
                  pack_bf16(__uint_as_float(o1[4 * gg]), __uint_as_float(o1[4 * gg + 1]));
              if (p.dr)
                *reinterpret_cast<uint32_t*>(p.dr + (rb + q_lo) * D + col) =
                    pack_bf16(__uint_as_float(o2[4 * gg]), __uint_as_float(o2[4 * gg + 1]));
            }
            if (q_hi < p.N) {
              *reinterpret_cast<uint32_t*>(p.dq + (rb + q_hi) * D + col) =
                  pack_bf16(__uint_as_float(o1[4 * gg + 2]), __uint_as_float(o1[4 * gg + 3]));
              if (p.dr)
                *reinterpret_cast<uint32_t*>(p.dr + (rb + q_hi) * D + col) =
                    pack_bf16(__uint_as_float(o2[4 * gg + 2]), __uint_as_float(o2[4 * gg + 3]));
            }
          }
        }
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == kBwdMmaWarp) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

// ---------------------------------------------------------------- dK, dV
template <int D>
struct BwdKVCfg {
  static constexpr int kCB = D / 64;
  static constexpr int kBlock = 128 * 128;        // [128 rows x 128 B]
  static constexpr int kDOBlock = 64 * 128;       // [64 rows x 128 B]
  static constexpr int kTileBytes = kCB * kBlock;  // K, V, [Q;R]
  static constexpr int kDOBytes = kCB * kDOBlock;  // dO (64 rows)
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kTileBytes;
  static constexpr int kOffQR = 2 * kTileBytes;
  static constexpr int kOffDO = kOffQR + kBwdStages * kTileBytes;
  static constexpr int kOffStat = kOffDO + kBwdStages * kDOBytes;  // per warp: 64 floats (its 16 queries)
  static constexpr int kOffBar = kOffStat + kBwdElemWarps * 16 * 16;
  static constexpr int kSmemBytes = kOffBar + 256 + 1024;
  // tensor memory: [A^T | S^T] [0,128), G^T of item i at 128 + 64 (i & 1) (two
  // buffers), dK [256,256+D), dV [256+D, 256+2D).  bf16 results: scale dA^T and
  // dS^T over the score columns, W_hat^T over its G^T.
  static constexpr uint32_t kColS = 0, kColG = 128, kColDK = 256, kColDV = 256 + D;
  static constexpr uint32_t kTmemCols = 512;
};

template <int D, bool HAS_R>
__global__ void __launch_bounds__(kBwdThreads, 1)
plx_bwd_kv_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap rmap,
                  const __grid_constant__ CUtensorMap omap, const __grid_constant__ CUtensorMap kmap,
                  const __grid_constant__ CUtensorMap vmap, const BwdParams p) {
  using Cfg = BwdKVCfg<D>;
  constexpr int NS = kBwdStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kOffBar);
  uint64_t* kv_full = bars;             // [1] K and V of this CTA's key tile landed
  uint64_t* q_full = bars + 1;          // [NS] [Q;R] and dO of a query tile landed
  uint64_t* q_empty = q_full + NS;      // [NS]
  uint64_t* s_full = q_empty + NS;      // [1] [A^T|S^T] and G^T in TMEM
  uint64_t* p_ready = s_full + 1;       // [1] W_hat^T, dA^T, dS^T written (one arrival per element-wise warp)
  uint64_t* o_done = p_ready + 1;       // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_done + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int per = p.B * p.Hkv;
  const int kt = static_cast<int>(blockIdx.x) / per;  // early key tiles see the most queries: first
  const int bg = static_cast<int>(blockIdx.x) % per;  // b * Hkv + g
  const int b = bg / p.Hkv, g = bg % p.Hkv;
  const int k0 = kt * kBwdBN;
  const int qt0 = p.causal ? k0 / kBwdBM : 0;
  const int n_qt = p.n_qtiles - qt0;
  const int n_items = p.G * n_qt;  // (query head, query tile) pairs, head-major

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(kv_full), 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(smem_u32(&q_full[s]), 1);
      mbar_init(smem_u32(&q_empty[s]), 1);
    }
    mbar_init(smem_u32(s_full), 1);
    mbar_init(smem_u32(p_ready), kBwdElemWarps);  // one arrival per element-wise warp
    mbar_init(smem_u32(o_done), 1);
    fence_barrier_init();
  }
  if (!HAS_R) {
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    for (int i = threadIdx.x; i < NS * Cfg::kCB * 4 * 16 * 8; i += kBwdThreads) {
      const int c16 = i & 7, row = (i >> 3) & 15, w = (i >> 7) & 3, cb = (i >> 9) % Cfg::kCB,
                s = (i >> 9) / Cfg::kCB;
      uint8_t* dst = smem + Cfg::kOffQR + s * Cfg::kTileBytes + cb * Cfg::kBlock + (32 * w + 16 + row) * 128 + c16 * 16;
      *reinterpret_cast<uint4*>(dst) = z;
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == kBwdMmaWarp) {
    tc::tmem_alloc(smem_u32(tmem_slot), Cfg::kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;

  if (warp == kBwdTmaWarp) {
    // ================================================================ TMA producer
    if (lane == 0) {
      {
        const uint32_t fb = smem_u32(kv_full);
        mbar_arrive_expect_tx(fb, 2 * Cfg::kTileBytes);
#pragma unroll
        for (int cb = 0; cb < Cfg::kCB; ++cb) {
          tma_load_3d(&kmap, smem_u32(smem + Cfg::kOffK + cb * Cfg::kBlock), fb, cb * 64, k0, bg);
          tma_load_3d(&vmap, smem_u32(smem + Cfg::kOffV + cb * Cfg::kBlock), fb, cb * 64, k0, bg);
        }
      }
      int issued = 0;
      for (int it = 0; it < n_items; ++it) {
        const int s = it % NS;
        if (it >= NS && !mbar_wait_sleep(smem_u32(&q_empty[s]), ((it / NS) - 1) & 1, kErrBwdLoad)) { ok = false; break; }
        const int hq = g * p.G + it / n_qt;
        const int q0 = (qt0 + it % n_qt) * kBwdBM;
        const int plane = b * p.Hq + hq;
        const uint32_t fb = smem_u32(&q_full[s]);
        mbar_arrive_expect_tx(fb, (HAS_R ? 2 : 1) * Cfg::kTileBytes / 2 + Cfg::kDOBytes);
        const uint32_t qr = smem_u32(smem + Cfg::kOffQR + s * Cfg::kTileBytes);
        const uint32_t dob = smem_u32(smem + Cfg::kOffDO + s * Cfg::kDOBytes);
#pragma unroll
        for (int wq = 0; wq < 4; ++wq)
#pragma unroll
          for (int cb = 0; cb < Cfg::kCB; ++cb) {
            const uint32_t dst = qr + cb * Cfg::kBlock + (32 * wq) * 128;
            tma_load_3d(&qmap, dst, fb, cb * 64, q0 + 16 * wq, plane);
            if (HAS_R) tma_load_3d(&rmap, dst + 16 * 128, fb, cb * 64, q0 + 16 * wq, plane);
            tma_load_3d(&omap, dob + cb * Cfg::kDOBlock + (16 * wq) * 128, fb, cb * 64, q0 + 16 * wq, plane);
          }
        issued = it + 1;
      }
      if (!ok) {
        mbar_wait(smem_u32(kv_full), 0, kErrBwdDrain);
        for (int it = max(0, issued - NS); it < issued; ++it) mbar_wait(smem_u32(&q_full[it % NS]), (it / NS) & 1, kErrBwdDrain);
      }
    }
  } else if (warp == kBwdMmaWarp) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = tc::idesc_bf16_f32(128, 128, 0, 0);  // K [Q;R]^T
      constexpr uint32_t idesc_g = tc::idesc_bf16_f32(128, kBwdBM, 0, 0);  // V dO^T
      constexpr uint32_t idesc_o = tc::idesc_bf16_f32(128, D, 0, 1);   // X^T Y, Y MN-major
      const uint64_t d_k = tc::smem_desc_sw128(smem_u32(smem + Cfg::kOffK), 16, 1024);
      const uint64_t d_v = tc::smem_desc_sw128(smem_u32(smem + Cfg::kOffV), 16, 1024);
      const uint64_t d_qr = tc::smem_desc_sw128(smem_u32(smem + Cfg::kOffQR), 16, 1024);
      const uint64_t d_do = tc::smem_desc_sw128(smem_u32(smem + Cfg::kOffDO), 16, 1024);
      const uint64_t d_qr_mn = tc::smem_desc_sw128(smem_u32(smem + Cfg::kOffQR), Cfg::kBlock, 1024);
      const uint64_t d_do_mn = tc::smem_desc_sw128(smem_u32(smem + Cfg::kOffDO), Cfg::kDOBlock, 1024);
      // Per item i, in issue order (the tensor pipe runs them in that order):
      // G^T(i+1) into the other G^T buffer, then after the element-wise pass
      // of i: dK(i) (the last reader of the score columns), [A^T|S^T](i+1),
      // dV(i).  The element-wise pass of i+1 waits only for dK(i) and the
      // scores of i+1; dV(i) and G^T(i+2) run during it.
      auto issue_s = [&](int it) {
        const uint64_t qr_off = static_cast<uint64_t>(it % NS) * (Cfg::kTileBytes >> 4);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint64_t koff = static_cast<uint64_t>(((ks >> 2) * Cfg::kBlock + (ks & 3) * 32) >> 4);
          tc::mma_ss(tmem + Cfg::kColS, d_k + koff, d_qr + qr_off + koff, idesc_s, ks > 0 ? 1u : 0u);
        }
      };
      auto issue_g = [&](int it) {
        const uint64_t do_off = static_cast<uint64_t>(it % NS) * (Cfg::kDOBytes >> 4);
        const uint32_t gcol = Cfg::kColG + 64 * static_cast<uint32_t>(it & 1);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint64_t koff_a = static_cast<uint64_t>(((ks >> 2) * Cfg::kBlock + (ks & 3) * 32) >> 4);
          const uint64_t koff_b = static_cast<uint64_t>(((ks >> 2) * Cfg::kDOBlock + (ks & 3) * 32) >> 4);
          tc::mma_ss(tmem + gcol, d_v + koff_a, d_do + do_off + koff_b, idesc_g, ks > 0 ? 1u : 0u);
        }
      };
      ok = mbar_wait(smem_u32(kv_full), 0, kErrBwdMma) && (n_items == 0 || mbar_wait(smem_u32(&q_full[0]), 0, kErrBwdMma));
      if (ok && n_items > 0) {
        tc::fence_after_sync();
        issue_s(0);
        issue_g(0);
        tc::commit(smem_u32(s_full));
      }
      for (int it = 0; it < n_items && ok; ++it) {
        const int s = it % NS;
        const bool more = it + 1 < n_items;
        if (more) {
          if (!mbar_wait(smem_u32(&q_full[(it + 1) % NS]), ((it + 1) / NS) & 1, kErrBwdMma)) { ok = false; break; }
          tc::fence_after_sync();
          issue_g(it + 1);
        }
        if (!mbar_wait(smem_u32(p_ready), it & 1, kErrBwdMma)) { ok = false; break; }
        tc::fence_after_sync();
        const uint64_t qr_off = static_cast<uint64_t>(s) * (Cfg::kTileBytes >> 4);
        const uint64_t do_off = static_cast<uint64_t>(s) * (Cfg::kDOBytes >> 4);
        // dK += [scale dA^T | dS^T] [Q ; R] (K = 128 stacked rows; the pairs of
        // stacked rows 32c..32c+15 sit at column 32c, of rows 32c+16.. at 32c+8)
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk)
          tc::mma_ts(tmem + Cfg::kColDK, tmem + Cfg::kColS + 32 * (kk >> 1) + 8 * (kk & 1),
                     d_qr_mn + qr_off + static_cast<uint64_t>((kk * 2048) >> 4), idesc_o, (it > 0 || kk > 0) ? 1u : 0u);
        if (more) {
          issue_s(it + 1);
          tc::commit(smem_u32(s_full));  // scores of i+1, and G^T(i+1) issued before
        }
        // dV += W_hat^T dO (K = 64 queries; the pairs of queries 16kk.. sit at G^T column 16kk)
        const uint32_t gcol = Cfg::kColG + 64 * static_cast<uint32_t>(it & 1);
#pragma unroll
        for (int kk = 0; kk < kBwdBM / 16; ++kk)
          tc::mma_ts(tmem + Cfg::kColDV, tmem + gcol + 16 * kk,
                     d_do_mn + do_off + static_cast<uint64_t>((kk * 2048) >> 4), idesc_o, (it > 0 || kk > 0) ? 1u : 0u);
        tc::commit(smem_u32(&q_empty[s]));
      }
      tc::commit(smem_u32(o_done));
      mbar_wait(smem_u32(o_done), 0, kErrBwdMma);
    }
  } else {
    // ================================================================ element-wise + epilogue
    // warp (wq, wp): keys 32wq..32wq+31 of the tile (thread = key: TMEM lane
    // 32wq + lane), queries 16wp..16wp+15 of each query tile
    const int wq = warp & 3, wp = warp >> 2;
    const int key = k0 + 32 * wq + lane;
    const uint32_t lane_base = static_cast<uint32_t>(32 * wq) << 16;
    const bool key_ok = key < p.N;
    // this warp's 16 queries, pair-interleaved: for queries (2i, 2i+1) the
    // float4s {L0, L1, F0, F1} and {G0, G1, D0, D1}, so that one load yields
    // the packed pairs the f32x2 arithmetic takes
    float* statf = reinterpret_cast<float*>(smem + Cfg::kOffStat) + warp * 64;
    const float4* stat = reinterpret_cast<const float4*>(statf);
    for (int it = 0; it < n_items; ++it) {
      const int hq = g * p.G + it / n_qt;
      const int q0 = (qt0 + it % n_qt) * kBwdBM + 16 * wp;  // first of this warp's queries
      const size_t rb = (static_cast<size_t>(b) * p.Hq + hq) * p.N;
      __syncwarp();
      if (lane < 16) {
        // per query: L = -lse log2(e), F = 1 + s_bar, G = g_bar, D = -Dd (rows past N: w = 0)
        const int q = q0 + lane;
        float L = -INFINITY, F = 1.f, G = 0.f, Dn = 0.f;
        if (q < p.N) {
          L = -p.lse[rb + q] * kLog2e;
          F = 1.f + (HAS_R ? p.sbar[rb + q] : 0.f);
          G = p.gbar[rb + q];
          Dn = -p.dd[rb + q];
        }
        float* sp = statf + (lane >> 1) * 8 + (lane & 1);
        sp[0] = L;
        sp[2] = F;
        sp[4] = G;
        sp[6] = Dn;
      }
      __syncwarp();
      const bool landed = mbar_wait_sleep(smem_u32(s_full), it & 1, kErrBwdElem);
      if (!__all_sync(0xffffffffu, landed)) { ok = false; break; }
      tc::fence_after_sync();
      // masks only where some (key, query) of this warp is out of the set:
      // keys past N, or (causal) a key of the warp after its first query
      const bool need_mask = (k0 + 32 * wq + 31 >= p.N) || (p.causal && k0 + 32 * wq + 31 > q0);
      // stacked columns 32wp..32wp+15 (q.k) and 32wp+16..32wp+31 (rho.k), G^T columns 16wp..16wp+15
      const uint32_t tsa = tmem + lane_base + Cfg::kColS + 32 * wp;
      const uint32_t tgw = tmem + lane_base + Cfg::kColG + 64 * static_cast<uint32_t>(it & 1) + 16 * wp;
      uint32_t ra[16], rs[16], rg[16];
      tc::ld_32x32b_x16(tsa, ra);
      tc::ld_32x32b_x16(tsa + 16, rs);
      tc::ld_32x32b_x16(tgw, rg);
      tc::wait_ld();
      // two queries at a time in packed f32x2 arithmetic:
      //   w = 2^(a scale log2e - lse log2e), f = 1 + s_bar - s,
      //   w_hat = w f,  dS = w (g_bar - g),  scale dA = (scale w)(g f + s g_bar - Dd)
      const uint64_t c_sl2 = f2(p.scale_log2, p.scale_log2), c_m1 = f2(-1.f, -1.f), c_sc = f2(p.scale, p.scale);
      uint32_t pw[8], pa[8], pd[8];
#pragma unroll
      for (int x = 0; x < 16; x += 2) {
        const float4 sa = stat[x], sb = stat[x + 1];  // {L0, L1, F0, F1}, {G0, G1, D0, D1} of queries x, x+1
        const uint64_t A = f2(__uint_as_float(ra[x]), __uint_as_float(ra[x + 1]));
        const uint64_t S = f2(__uint_as_float(rs[x]), __uint_as_float(rs[x + 1]));
        const uint64_t Gv = f2(__uint_as_float(rg[x]), __uint_as_float(rg[x + 1]));
        const uint64_t X = f2_fma(A, c_sl2, f2(sa.x, sa.y));
        float w0 = ex2(f2_lo(X)), w1 = ex2(f2_hi(X));
        if (need_mask) {
          const int q = q0 + x;
          if (!key_ok || (p.causal && key > q)) w0 = 0.f;
          if (!key_ok || (p.causal && key > q + 1)) w1 = 0.f;
        }
        const uint64_t W = f2(w0, w1);
        const uint64_t Gb = f2(sb.x, sb.y);
        const uint64_t F = f2_fma(S, c_m1, f2(sa.z, sa.w));                    // 1 + s_bar - s
        const uint64_t WH = f2_mul(W, F);
        const uint64_t DS = f2_mul(W, f2_fma(Gv, c_m1, Gb));                    // w (g_bar - g)
        const uint64_t U = f2_fma(Gv, F, f2_fma(S, Gb, f2(sb.z, sb.w)));       // g f + s g_bar - Dd
        const uint64_t DA = f2_mul(f2_mul(W, c_sc), U);
        pw[x >> 1] = pack_bf16(f2_lo(WH), f2_hi(WH));
        pa[x >> 1] = pack_bf16(f2_lo(DA), f2_hi(DA));
        pd[x >> 1] = pack_bf16(f2_lo(DS), f2_hi(DS));
      }
      // bf16 pairs over this warp's own fp32 columns (already read)
      tc::st_32x32b_x8(tgw, pw);
      tc::st_32x32b_x8(tsa, pa);
      tc::st_32x32b_x8(tsa + 8, pd);
      tc::wait_st();
      tc::fence_before_sync();
      __syncwarp();  // every lane's stores are complete: one lane arrives for the warp
      if (lane == 0) mbar_arrive(smem_u32(p_ready));
    }
    if (ok) {
      const bool done = mbar_wait_sleep(smem_u32(o_done), 0, kErrBwdElem);
      if (__all_sync(0xffffffffu, done)) {
        tc::fence_after_sync();
        const size_t row = static_cast<size_t>(bg) * p.N + key;
        // this warp's quarter of the columns: [wp * D/4, (wp + 1) * D/4)
#pragma unroll
        for (int which = 0; which < 2; ++which) {
          const uint32_t col = which == 0 ? Cfg::kColDK : Cfg::kColDV;
          __nv_bfloat16* dst = (which == 0 ? p.dk : p.dv) + row * D;
#pragma unroll
          for (int ch = 0; ch < D / 64; ++ch) {
            const int cbase = wp * (D / 4) + 16 * ch;
            uint32_t v[16];
            tc::ld_32x32b_x16(tmem + lane_base + col + cbase, v);
            tc::wait_ld();
            if (key_ok) {
              uint4 lo, hi;
              lo.x = pack_bf16(__uint_as_float(v[0]), __uint_as_float(v[1]));
              lo.y = pack_bf16(__uint_as_float(v[2]), __uint_as_float(v[3]));
              lo.z = pack_bf16(__uint_as_float(v[4]), __uint_as_float(v[5]));
              lo.w = pack_bf16(__uint_as_float(v[6]), __uint_as_float(v[7]));
              hi.x = pack_bf16(__uint_as_float(v[8]), __uint_as_float(v[9]));
              hi.y = pack_bf16(__uint_as_float(v[10]), __uint_as_float(v[11]));
              hi.z = pack_bf16(__uint_as_float(v[12]), __uint_as_float(v[13]));
              hi.w = pack_bf16(__uint_as_float(v[14]), __uint_as_float(v[15]));
              *reinterpret_cast<uint4*>(dst + cbase) = lo;
              *reinterpret_cast<uint4*>(dst + cbase + 8) = hi;
            }
          }
        }
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == kBwdMmaWarp) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

}  // namespace plx
