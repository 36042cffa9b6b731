// plx_fwd.cuh -- Parallax prefill / full-sequence forward on sm_100a.
//
// Method (gist.science, "Technical overview: Parallax - parameterized local
// linear attention for language modeling", section "Method: Parallax / Core
// mechanism"): out_i = o_SA_i - Sigma_i rho_i.  Streamed as in
// news.chathome.org, "Parallax: a parameterized local linear attention ...",
// section "Hardware argument": two score branches share the online max, the
// rescale factor and the K/V tiles.
//
// Design (one CTA per pair of 64-query tiles, 320 threads):
//   * A query tile and its probes form ONE stacked MMA operand [Q;R] of 128
//     rows, interleaved in blocks of 16: rows 32w..32w+15 hold queries
//     16w..16w+15 and rows 32w+16..32w+31 hold their probes.  One tcgen05 MMA
//     (M=128, N=128 keys, K=d) gives both branches, a = q.k in TMEM lanes
//     32w+r and s = rho.k in lanes 32w+16+r.  A 16x256b tensor-memory load
//     at lane 32w and another at 32w+16 hand every thread a and s for the
//     SAME (query, key) pairs, so the shared softmax needs no data exchange.
//   * The value product uses the same stacking: P (bf16) is written over the
//     a rows and P*S over the s rows of the score columns in TMEM, and one
//     MMA [P ; P*S] x V (A from tensor memory) accumulates O1 = sum p v and
//     O2 = sum p s v in the matching rows of one 128-lane accumulator.
//   * Two query tiles share every K/V tile: heads (h, h+1) of one KV group at
//     the same rows when the group size is even, otherwise rows (q0, q0+64)
//     of one head.  Tensor memory: [S0 | O0 | S1 | O1], 128 columns each.
//   * Warps 0-3 and 4-7: softmax + epilogue of tile 0 and tile 1;
//     warp 8: TMA loads (Q/R once, K/V ring); warp 9: TMEM allocation and
//     the single thread that issues every MMA (warps 10-11 only complete the
//     third warpgroup, so that setmaxnreg can move registers from it to the
//     softmax warps), in the order
//     PV0(j), S0(j+1), PV1(j), S1(j+1): each tile's next scores come right
//     after its value MMA, so each softmax overlaps the other tile's MMAs.
//     One M=128 N=128 MMA takes ~64 tensor cycles and a thread needs a large
//     part of that to issue one, so descriptors are precomputed and each MMA
//     only adds a constant to the start-address field.  Each softmax hands
//     over P in two 64-key halves so the first half of its value MMA runs
//     while it computes the second.
//   * Persistent: one CTA per SM walks the work units (tile pairs, longest
//     causal rows first) in steps of the grid size.  The K/V ring and every
//     barrier phase carry on across units; the load warp fetches the next
//     unit's Q/R as soon as the last score MMA of the current unit has been
//     issued, the next unit's score MMAs overlap this unit's epilogue, and
//     its first value MMA waits only until the epilogue has read O.
//   * The running max is updated lazily: O is rescaled in tensor memory only
//     when a row max grows by more than 2^8 (so p <= 256 before the final
//     normalisation, which bf16 P holds without loss of relative precision).
#pragma once

#include "plx_ptx.cuh"
#include "plx_tcgen05.cuh"

namespace plx {

constexpr int kFwdBM = 64;        // queries per tile (128 stacked rows with their probes)
constexpr int kFwdBN = 128;       // keys per K/V tile
constexpr int kFwdThreads = 384;  // 8 softmax warps, TMA warp, MMA warp, 2 idle warps (3 warpgroups)
// registers per thread after setmaxnreg: the two softmax warpgroups gain
// what the load/MMA warpgroup gives up (3 x 128 x 168 = 2 x 128 x 200 + 128 x 104)
constexpr int kFwdRegsSoftmax = 200;
constexpr int kFwdRegsOther = 104;
constexpr int kFwdTmaWarp = 8;
constexpr int kFwdMmaWarp = 9;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int D>
struct FwdCfg {
  static constexpr int kCB = D / 64;                 // 128-byte column blocks per row
  static constexpr int kBlock = 128 * 128;           // bytes of one [128 rows x 128 B] block
  static constexpr int kQRBytes = kCB * kBlock;      // stacked [Q;R] tile
  static constexpr int kKVBytes = kCB * kBlock;      // one K or V tile (128 keys)
  static constexpr int kStages = D == 128 ? 2 : 3;
  static constexpr int kOffQR = 0;
  static constexpr int kOffK = 2 * kQRBytes;
  static constexpr int kOffV = kOffK + kStages * kKVBytes;
  static constexpr int kOffOut = kOffV + kStages * kKVBytes;     // bf16 output staging for TMA stores
  static constexpr int kOutWarpBytes = kCB * 16 * 128;              // 16 rows per softmax warp
  static constexpr int kOffBar = kOffOut + 8 * kOutWarpBytes;
  static constexpr int kSmemBytes = kOffBar + 256 + 1024;  // barriers + alignment slack
  static constexpr uint32_t kTmemCols = 512;
};

struct FwdParams {
  __nv_bfloat16* out;  // [B, Hq, N, D]
  float* lse;          // [B, Hq, N] or nullptr
  int B, Hq, Hkv, N, G;
  int pair_heads;      // 1: tiles are heads (2p, 2p+1) at rows 64*qb; 0: rows 128*qb (+64) of head p
  int n_pairs;         // Hq / 2 or Hq
  int n_qblocks;       // ceil(N/64) or ceil(N/128)
  int num_units;       // B * n_pairs * n_qblocks
  int causal;
  float scale_log2;    // scale * log2(e)
  float* sbar;         // [B, Hq, N] s_bar = c / l (training forward only)
  __nv_bfloat16* obar; // o_bar (training forward only; written by TMA, by this pointer only for
                       // the last rows of a packed sequence)
  // variable-length packed sequences (nullptr: fixed length N).  Then q, r,
  // out are [total, Hq, D] and k, v [total, Hkv, D] (token-major; the tensor
  // maps take a head as the plane and a token as the row), sequence b is rows
  // cu_seqlens[b] .. cu_seqlens[b+1]-1, N is the longest length, and lse /
  // sbar are [Hq, total].
  const int* cu_seqlens;
  int total;
  long long lse_stride;  // N (fixed length) or total (packed)
  // partial-state forward only: [B, Hq, N, 2D + 4] fp32, per query row the
  // record m (log2 units), l, c, pad, O1[D], O2[D] of the split-KV merge
  float* partial;
};

// What the softmax warps write per unit: the output (and lse), the output plus
// o_bar and s_bar for the backward, or the unnormalised partial state of each
// row over this call's keys (context-parallel prefill merges those).
constexpr int kFwdModeOut = 0, kFwdModeTrain = 1, kFwdModePartial = 2;

template <int D, bool HAS_R, int MODE>
__global__ void __launch_bounds__(kFwdThreads, 1)
plx_fwd_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap rmap,
               const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
               const __grid_constant__ CUtensorMap omap, const __grid_constant__ CUtensorMap amap,
               const FwdParams p) {
  using Cfg = FwdCfg<D>;
  constexpr int NS = Cfg::kStages;
  constexpr bool SAVE_AUX = MODE == kFwdModeTrain;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kOffBar);
  uint64_t* qr_full = bars;             // [2]
  uint64_t* qr_empty = bars + 2;        // [1] last score MMA of a unit issued and done
  uint64_t* k_full = bars + 3;          // [NS]
  uint64_t* k_empty = k_full + NS;      // [NS]
  uint64_t* v_full = k_empty + NS;      // [NS]
  uint64_t* v_empty = v_full + NS;      // [NS]
  uint64_t* s_full = v_empty + NS;      // [2]
  uint64_t* p_ready = s_full + 2;       // [2 tiles][2 halves]
  uint64_t* o_done = p_ready + 4;       // [2]
  uint64_t* o_free = o_done + 2;        // [2] epilogue has read O (one arrival per softmax warp)
  uint64_t* fin = o_free + 2;           // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work units: index u -> (b, head pair / head, query block), longest
  // causal rows first; CTA c takes u = c, c + gridDim.x, ...
  // (packed sequences: a unit whose query block starts past its sequence is
  // empty, nkv = 0, and every role skips it the same way)
  struct Unit {
    int b, hp, qb, nkv;
    int N, base;  // the sequence's length and first row
  };
  auto unit_of = [&](int u) {
    Unit w;
    const int per = p.B * p.n_pairs;
    w.qb = p.n_qblocks - 1 - u / per;
    const int rem = u % per;
    w.b = rem / p.n_pairs;
    w.hp = rem % p.n_pairs;
    w.base = 0;
    w.N = p.N;
    if (p.cu_seqlens) {  // clamped so that no row outside [0, total) is ever addressed
      w.base = min(max(__ldg(p.cu_seqlens + w.b), 0), p.total);
      w.N = min(max(__ldg(p.cu_seqlens + w.b + 1) - w.base, 0), min(p.total - w.base, p.N));
    }
    const int first_row = p.pair_heads ? w.qb * kFwdBM : 2 * w.qb * kFwdBM;
    const int last_row = p.pair_heads ? w.qb * kFwdBM + kFwdBM - 1 : (2 * w.qb + 2) * kFwdBM - 1;
    const int qmax = min(w.N - 1, last_row);
    const int nkv_all = (w.N + kFwdBN - 1) / kFwdBN;
    w.nkv = first_row >= w.N ? 0 : (p.causal ? min(nkv_all, qmax / kFwdBN + 1) : nkv_all);
    return w;
  };
  // tile t in {0, 1} of a unit: query head and first query row
  auto head_of = [&](const Unit& w, int t) { return p.pair_heads ? 2 * w.hp + t : w.hp; };
  auto row0_of = [&](const Unit& w, int t) { return p.pair_heads ? w.qb * kFwdBM : (2 * w.qb + t) * kFwdBM; };
  // tensor-map plane of a query head and of its KV head (packed: the head alone)
  auto qplane_of = [&](const Unit& w, int t) { return p.cu_seqlens ? head_of(w, t) : w.b * p.Hq + head_of(w, t); };
  auto kvplane_of = [&](const Unit& w) {
    return p.cu_seqlens ? head_of(w, 0) / p.G : w.b * p.Hkv + head_of(w, 0) / p.G;
  };

  if (threadIdx.x == 0) {
    // arrivals per phase: p_ready and o_free get one arrival from each of the
    // 4 warps of a softmax warpgroup; every other barrier one arrival (+ TMA
    // bytes / a commit)
    for (int i = 0; i < 3 + 4 * NS + 11; ++i) {
      uint64_t* bp = &bars[i];
      const bool wg = (bp >= &p_ready[0] && bp <= &p_ready[3]) || bp == &o_free[0] || bp == &o_free[1];
      mbar_init(smem_u32(bp), wg ? 4u : 1u);
    }
    fence_barrier_init();
  }
  if (!HAS_R) {
    // rho = 0: zero the probe rows of both stacked tiles once (TMA loads only Q).
    uint4 z = make_uint4(0u, 0u, 0u, 0u);
    for (int i = threadIdx.x; i < 2 * Cfg::kCB * 4 * 16 * 8; i += kFwdThreads) {
      const int c16 = i & 7, row = (i >> 3) & 15, w = (i >> 7) & 3, cb = (i >> 9) % Cfg::kCB,
                t = (i >> 9) / Cfg::kCB;
      uint8_t* dst = smem + Cfg::kOffQR + t * Cfg::kQRBytes + cb * Cfg::kBlock + (32 * w + 16 + row) * 128 + c16 * 16;
      *reinterpret_cast<uint4*>(dst) = z;
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == kFwdMmaWarp) {
    tc::tmem_alloc(smem_u32(tmem_slot), Cfg::kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  // tensor-memory columns: [S0 | O0 | S1 | O1]
  auto col_s = [](int t) { return static_cast<uint32_t>(256 * t); };
  auto col_o = [](int t) { return static_cast<uint32_t>(256 * t + 128); };
  bool ok = true;

  if (warp >= kFwdTmaWarp) {
    // warpgroup 2 (load, MMA and two idle warps) gives registers to the softmax warpgroups
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kFwdRegsOther));
  if (warp == kFwdTmaWarp) {
    // ================================================================ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&qmap);
      if (HAS_R) tma_prefetch_desc(&rmap);
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&vmap);
      int kv = 0;        // K/V tiles issued so far: ring stage kv % NS, phase (kv / NS) & 1
      int n_unit = 0;    // units whose Q/R were issued
      int issued_k = 0, issued_v = 0;
      for (int u = blockIdx.x; u < p.num_units && ok; u += gridDim.x) {
        const Unit w = unit_of(u);
        if (w.nkv == 0) continue;
        // the previous unit's last score MMA must have read Q/R
        if (n_unit > 0 && !mbar_wait(smem_u32(qr_empty), (n_unit - 1) & 1, kErrFwdLoad)) { ok = false; break; }
        for (int t = 0; t < 2; ++t) {
          const uint32_t fb = smem_u32(&qr_full[t]);
          mbar_arrive_expect_tx(fb, HAS_R ? Cfg::kQRBytes : Cfg::kQRBytes / 2);
          const uint32_t base = smem_u32(smem + Cfg::kOffQR + t * Cfg::kQRBytes);
          const int plane = qplane_of(w, t);
          const int row0 = w.base + row0_of(w, t);
#pragma unroll
          for (int wq = 0; wq < 4; ++wq)
#pragma unroll
            for (int cb = 0; cb < Cfg::kCB; ++cb) {
              const uint32_t dst = base + cb * Cfg::kBlock + (32 * wq) * 128;
              tma_load_3d(&qmap, dst, fb, cb * 64, row0 + 16 * wq, plane);
              if (HAS_R) tma_load_3d(&rmap, dst + 16 * 128, fb, cb * 64, row0 + 16 * wq, plane);
            }
        }
        const int plane_kv = kvplane_of(w);
        for (int j = 0; j < w.nkv; ++j, ++kv) {
          const int s = kv % NS;
          if (kv >= NS && !mbar_wait(smem_u32(&k_empty[s]), ((kv / NS) - 1) & 1, kErrFwdLoad)) { ok = false; break; }
          {
            const uint32_t fb = smem_u32(&k_full[s]);
            mbar_arrive_expect_tx(fb, Cfg::kKVBytes);
            const uint32_t dst = smem_u32(smem + Cfg::kOffK + s * Cfg::kKVBytes);
#pragma unroll
            for (int cb = 0; cb < Cfg::kCB; ++cb)
              tma_load_3d(&kmap, dst + cb * Cfg::kBlock, fb, cb * 64, w.base + j * kFwdBN, plane_kv);
            issued_k = kv + 1;
          }
          if (kv >= NS && !mbar_wait(smem_u32(&v_empty[s]), ((kv / NS) - 1) & 1, kErrFwdLoad)) { ok = false; break; }
          {
            const uint32_t fb = smem_u32(&v_full[s]);
            mbar_arrive_expect_tx(fb, Cfg::kKVBytes);
            const uint32_t dst = smem_u32(smem + Cfg::kOffV + s * Cfg::kKVBytes);
#pragma unroll
            for (int cb = 0; cb < Cfg::kCB; ++cb)
              tma_load_3d(&vmap, dst + cb * Cfg::kBlock, fb, cb * 64, w.base + j * kFwdBN, plane_kv);
            issued_v = kv + 1;
          }
        }
        ++n_unit;
      }
      if (!ok) {  // let every issued load land before the CTA can exit
        if (n_unit > 0)
          for (int t = 0; t < 2; ++t) mbar_wait(smem_u32(&qr_full[t]), (n_unit - 1) & 1, kErrFwdDrain);
        for (int j = max(0, issued_k - NS); j < issued_k; ++j)
          mbar_wait(smem_u32(&k_full[j % NS]), (j / NS) & 1, kErrFwdDrain);
        for (int j = max(0, issued_v - NS); j < issued_v; ++j)
          mbar_wait(smem_u32(&v_full[j % NS]), (j / NS) & 1, kErrFwdDrain);
      }
    }
  } else if (warp == kFwdMmaWarp) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = tc::idesc_bf16_f32(128, kFwdBN, 0, 0);  // [Q;R] x K^T, both K-major
      constexpr uint32_t idesc_o = tc::idesc_bf16_f32(128, D, 0, 1);       // [P;PS] x V, V MN-major
      constexpr uint64_t kStageStep = Cfg::kKVBytes >> 4;                  // descriptor units
      constexpr uint64_t kTileStep = Cfg::kQRBytes >> 4;
      // base descriptors; each MMA adds a constant to the start-address field
      const uint64_t d_qr = tc::smem_desc_sw128(smem_u32(smem + Cfg::kOffQR), 16, 1024);
      const uint64_t d_k = tc::smem_desc_sw128(smem_u32(smem + Cfg::kOffK), 16, 1024);
      const uint64_t d_v = tc::smem_desc_sw128(smem_u32(smem + Cfg::kOffV), Cfg::kBlock, 1024);

      // S_t = [Q;R]_t K^T of the K/V tile in ring stage s, into tile t's score columns
      auto issue_s = [&](int t, int s) {
        const uint64_t da = d_qr + t * kTileStep;
        const uint64_t db = d_k + s * kStageStep;
        const uint32_t dst = tmem + col_s(t);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint64_t koff = static_cast<uint64_t>(((ks >> 2) * Cfg::kBlock + (ks & 3) * 32) >> 4);
          tc::mma_ss(dst, da + koff, db + koff, idesc_s, ks > 0 ? 1u : 0u);
        }
        tc::commit(smem_u32(&s_full[t]));
      };
      // O_t (+)= [P;PS]_t V for keys 64h..64h+63 of global tile g, once that half of P is ready
      auto issue_pv = [&](int t, int g, int h, bool first) -> bool {
        if (!mbar_wait(smem_u32(&p_ready[2 * t + h]), g & 1, kErrFwdMma)) return false;
        tc::fence_after_sync();
        const uint64_t db = d_v + (g % NS) * kStageStep;
        const uint32_t a = tmem + col_s(t), dst = tmem + col_o(t);
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          const int kk = 4 * h + k4;
          tc::mma_ts(dst, a + kk * 8, db + static_cast<uint64_t>((kk * 2048) >> 4), idesc_o,
                     (!first || kk > 0) ? 1u : 0u);
        }
        return true;
      };

      int kv = 0;       // global K/V tile index of the current unit's first tile
      int n_unit = 0;
      for (int u = blockIdx.x; u < p.num_units && ok; u += gridDim.x) {
        const Unit w = unit_of(u);
        if (w.nkv == 0) continue;
        const uint32_t uph = n_unit & 1;
        ok = mbar_wait(smem_u32(&qr_full[0]), uph, kErrFwdMma) && mbar_wait(smem_u32(&qr_full[1]), uph, kErrFwdMma) &&
             mbar_wait(smem_u32(&k_full[kv % NS]), (kv / NS) & 1, kErrFwdMma);
        if (!ok) break;
        tc::fence_after_sync();
        // The previous unit's PV(last) precede these in issue order, so they
        // overwrite its last P only after it was read.
        issue_s(0, kv % NS);
        issue_s(1, kv % NS);
        tc::commit(smem_u32(&k_empty[kv % NS]));
        if (w.nkv == 1) tc::commit(smem_u32(qr_empty));
        for (int j = 0; j < w.nkv && ok; ++j) {
          const int g = kv + j;
          const int s = g % NS;
          const bool more = j + 1 < w.nkv;
          if (!mbar_wait(smem_u32(&v_full[s]), (g / NS) & 1, kErrFwdMma)) { ok = false; break; }
          // a unit's first PV overwrites O: the previous unit's epilogue must have read it
          if (j == 0 && n_unit > 0 && !mbar_wait(smem_u32(&o_free[0]), (n_unit - 1) & 1, kErrFwdMma)) { ok = false; break; }
          if (!issue_pv(0, g, 0, j == 0) || !issue_pv(0, g, 1, j == 0)) { ok = false; break; }
          if (more) {
            // S0 of the next tile follows PV0 in issue order: it overwrites P0 only after it was read
            if (!mbar_wait(smem_u32(&k_full[(g + 1) % NS]), ((g + 1) / NS) & 1, kErrFwdMma)) { ok = false; break; }
            tc::fence_after_sync();
            issue_s(0, (g + 1) % NS);
          }
          if (j == 0 && n_unit > 0 && !mbar_wait(smem_u32(&o_free[1]), (n_unit - 1) & 1, kErrFwdMma)) { ok = false; break; }
          if (!issue_pv(1, g, 0, j == 0) || !issue_pv(1, g, 1, j == 0)) { ok = false; break; }
          tc::commit(smem_u32(&v_empty[s]));
          if (more) {
            issue_s(1, (g + 1) % NS);
            tc::commit(smem_u32(&k_empty[(g + 1) % NS]));
            if (j + 2 == w.nkv) tc::commit(smem_u32(qr_empty));  // last score MMAs of the unit
          } else {
            tc::commit(smem_u32(&o_done[0]));
            tc::commit(smem_u32(&o_done[1]));
          }
        }
        kv += w.nkv;
        ++n_unit;
      }
      // Every MMA issued must be complete before tensor memory is released.
      tc::commit(smem_u32(&fin[0]));
      mbar_wait(smem_u32(&fin[0]), 0, kErrFwdMma);
    }
  }
    tc::fence_before_sync();
    asm volatile("bar.sync 1, %0;" ::"n"(kFwdThreads) : "memory");  // every role is done
    if (warp == kFwdMmaWarp) {
      tc::fence_after_sync();
      tc::tmem_dealloc(tmem, Cfg::kTmemCols);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kFwdRegsSoftmax));
    // ================================================================ softmax + epilogue
    const int t = warp >> 2;     // query tile
    const int wq = warp & 3;     // TMEM lane quadrant
    const int c4 = lane & 3;
    const uint32_t lane_a = static_cast<uint32_t>(32 * wq) << 16;
    const uint32_t lane_s = static_cast<uint32_t>(32 * wq + 16) << 16;
    const uint32_t ta = tmem + lane_a + col_s(t);
    const uint32_t ts = tmem + lane_s + col_s(t);
    const uint32_t to1 = tmem + lane_a + col_o(t);
    const uint32_t to2 = tmem + lane_s + col_o(t);
    int kv = 0, n_unit = 0;
    for (int u = blockIdx.x; u < p.num_units && ok; u += gridDim.x) {
      const Unit w = unit_of(u);
      if (w.nkv == 0) continue;
      const int q0 = row0_of(w, t);
      const int q_lo = q0 + 16 * wq + (lane >> 2);
      const int q_hi = q_lo + 8;
      float m_lo = -INFINITY, m_hi = -INFINITY;
      // this thread's column share: l = sum p (fp32, also gives lse), c = sum of
      // the bf16-rounded p*s the value MMA consumes (so that O2 and c agree)
      float l_lo = 0.f, l_hi = 0.f, c_lo = 0.f, c_hi = 0.f;

      for (int j = 0; j < w.nkv; ++j) {
        const int g = kv + j;
        // warp-uniform: the .sync.aligned tensor-memory accesses below need every lane
        const bool landed = mbar_wait(smem_u32(&s_full[t]), g & 1, kErrFwdSoftmax);
        if (!__all_sync(0xffffffffu, landed)) { ok = false; break; }
        tc::fence_after_sync();
        uint32_t ra[64], rs[64];
        tc::ld_16x256b_x8(ta, *reinterpret_cast<uint32_t(*)[32]>(&ra[0]));
        tc::ld_16x256b_x8(ta + 64, *reinterpret_cast<uint32_t(*)[32]>(&ra[32]));
        tc::wait_ld();
        // the probe scores are needed only after the row max: their load
        // overlaps the max reduction (the next wait::ld collects it)
        if (HAS_R) {
          tc::ld_16x256b_x8(ts, *reinterpret_cast<uint32_t(*)[32]>(&rs[0]));
          tc::ld_16x256b_x8(ts + 64, *reinterpret_cast<uint32_t(*)[32]>(&rs[32]));
        }
        // register i: half h = i/32, rep g = (i%32)/4, e = i%4;
        // key = 64h + 8g + 2*c4 + (e&1); row lo for e < 2, row hi for e >= 2.
        // Masked scores become -inf in place; the max is taken on raw q.k and
        // scaled afterwards (scale_log2 > 0), and the scale folds into exp2's FMA.
        const int kbase = j * kFwdBN;
        const bool need_mask = (p.causal && kbase + kFwdBN - 1 > q0) || (kbase + kFwdBN > w.N);
        if (need_mask) {
#pragma unroll
          for (int i = 0; i < 64; ++i) {
            const int key = kbase + 64 * (i >> 5) + 8 * ((i & 31) >> 2) + 2 * c4 + (i & 1);
            const int q = (i & 2) ? q_hi : q_lo;
            const bool valid = key < w.N && (!p.causal || key <= q);
            if (!valid) ra[i] = 0xFF800000u;  // -inf
          }
        }
        // row maxima: four running three-input maxima per row (short chains)
        float tl[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        float th[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int gg = 0; gg < 16; ++gg) {
          tl[gg & 3] = fmax3(tl[gg & 3], __uint_as_float(ra[4 * gg]), __uint_as_float(ra[4 * gg + 1]));
          th[gg & 3] = fmax3(th[gg & 3], __uint_as_float(ra[4 * gg + 2]), __uint_as_float(ra[4 * gg + 3]));
        }
        float mx_lo = fmaxf(fmax3(tl[0], tl[1], tl[2]), tl[3]);
        float mx_hi = fmaxf(fmax3(th[0], th[1], th[2]), th[3]);
        mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 1));
        mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 1));
        mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 2)) * p.scale_log2;
        mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 2)) * p.scale_log2;
        const bool grow = mx_lo > m_lo + kRescaleThreshold || mx_hi > m_hi + kRescaleThreshold;
        if (__any_sync(0xffffffffu, grow)) {
          const float mn_lo = fmaxf(m_lo, mx_lo), mn_hi = fmaxf(m_hi, mx_hi);
          const float al_lo = mn_lo == -INFINITY ? 1.f : ex2(m_lo - mn_lo);
          const float al_hi = mn_hi == -INFINITY ? 1.f : ex2(m_hi - mn_hi);
          l_lo *= al_lo; c_lo *= al_lo; l_hi *= al_hi; c_hi *= al_hi;
          m_lo = mn_lo; m_hi = mn_hi;
          if (j > 0) {  // the unit's first PV starts O from zero
            // O rows of this warp: O1 at the a lanes, O2 at the s lanes; PV(j-1)
            // has completed (it precedes S(j) in the MMA stream).
#pragma unroll 1
            for (int ch = 0; ch < D / 16; ++ch) {
              uint32_t o1[8], o2[8];
              tc::ld_16x256b_x2(to1 + 16 * ch, o1);
              tc::ld_16x256b_x2(to2 + 16 * ch, o2);
              tc::wait_ld();
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const float al = (i & 2) ? al_hi : al_lo;
                o1[i] = __float_as_uint(__uint_as_float(o1[i]) * al);
                o2[i] = __float_as_uint(__uint_as_float(o2[i]) * al);
              }
              tc::st_16x256b_x2(to1 + 16 * ch, o1);
              tc::st_16x256b_x2(to2 + 16 * ch, o2);
            }
          }
        }
        if (HAS_R) tc::wait_ld();
        const float mu_lo = m_lo == -INFINITY ? 0.f : m_lo;
        const float mu_hi = m_hi == -INFINITY ? 0.f : m_hi;
        // p = 2^(a*scale*log2e - m) with the scale folded into one packed FMA per
        // row pair; l from fp32 p, c from the rounded p*s.
        const uint64_t sl2 = f2(p.scale_log2, p.scale_log2);
        const uint64_t nmu_lo = f2(-mu_lo, -mu_lo), nmu_hi = f2(-mu_hi, -mu_hi);
        uint64_t ls_lo = 0, ls_hi = 0, cs_lo = 0, cs_hi = 0;  // packed partial sums (0 bits = +0.0f)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t pp[16], pq[16];
#pragma unroll
          for (int gg = 0; gg < 8; ++gg) {
            const int i = 32 * hf + 4 * gg;
            const uint64_t xl = f2_fma(f2(__uint_as_float(ra[i]), __uint_as_float(ra[i + 1])), sl2, nmu_lo);
            const uint64_t xh = f2_fma(f2(__uint_as_float(ra[i + 2]), __uint_as_float(ra[i + 3])), sl2, nmu_hi);
            const uint64_t pl = f2(ex2(f2_lo(xl)), ex2(f2_hi(xl)));
            const uint64_t ph = f2(ex2(f2_lo(xh)), ex2(f2_hi(xh)));
            ls_lo = f2_add(ls_lo, pl);
            ls_hi = f2_add(ls_hi, ph);
            pp[2 * gg] = pack_bf16(f2_lo(pl), f2_hi(pl));
            pp[2 * gg + 1] = pack_bf16(f2_lo(ph), f2_hi(ph));
            if (HAS_R) {
              const uint64_t sl = f2_mul(pl, f2(__uint_as_float(rs[i]), __uint_as_float(rs[i + 1])));
              const uint64_t sh = f2_mul(ph, f2(__uint_as_float(rs[i + 2]), __uint_as_float(rs[i + 3])));
              const uint32_t wl = pack_bf16(f2_lo(sl), f2_hi(sl));
              const uint32_t wh = pack_bf16(f2_lo(sh), f2_hi(sh));
              pq[2 * gg] = wl;
              pq[2 * gg + 1] = wh;
              cs_lo = f2_add(cs_lo, f2(bf16_lo(wl), bf16_hi(wl)));
              cs_hi = f2_add(cs_hi, f2(bf16_lo(wh), bf16_hi(wh)));
            }
          }
          tc::st_16x128b_x8(ta + 32 * hf, pp);
          // rho = 0: the probe rows of S are exact zeros, which read as bf16 zeros
          if (HAS_R) tc::st_16x128b_x8(ts + 32 * hf, pq);
          tc::wait_st();
          tc::fence_before_sync();
          __syncwarp();  // every lane's stores are complete: one lane arrives for the warp
          if (lane == 0) mbar_arrive(smem_u32(&p_ready[2 * t + hf]));
        }
        l_lo += f2_lo(ls_lo) + f2_hi(ls_lo);
        l_hi += f2_lo(ls_hi) + f2_hi(ls_hi);
        c_lo += f2_lo(cs_lo) + f2_hi(cs_lo);
        c_hi += f2_lo(cs_hi) + f2_hi(cs_hi);
      }
      if (!ok) break;

      // ---- epilogue: out = O1/l - (O2/l - (c/l)(O1/l)), lse = m + log2(l) (in ln units)
      const bool done = mbar_wait(smem_u32(&o_done[t]), n_unit & 1, kErrFwdSoftmax);
      if (!__all_sync(0xffffffffu, done)) { ok = false; break; }
      tc::fence_after_sync();
      l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 1);
      l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 2);
      l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 1);
      l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 2);
      c_lo += __shfl_xor_sync(0xffffffffu, c_lo, 1);
      c_lo += __shfl_xor_sync(0xffffffffu, c_lo, 2);
      c_hi += __shfl_xor_sync(0xffffffffu, c_hi, 1);
      c_hi += __shfl_xor_sync(0xffffffffu, c_hi, 2);
      if constexpr (MODE == kFwdModePartial) {
        // This warp's 16 rows as partial states over this call's keys: O1 and
        // O2 straight from tensor memory (relative to m, as accumulated),
        // m = -inf for a row that saw no key.  Fixed-length layout only.
        constexpr int PF = 2 * D + 4;
        const size_t plane = static_cast<size_t>(qplane_of(w, t));
        const bool live_lo = q_lo < w.N, live_hi = q_hi < w.N;
        float* rec_lo = p.partial + (plane * p.N + static_cast<size_t>(live_lo ? q_lo : 0)) * PF;
        float* rec_hi = p.partial + (plane * p.N + static_cast<size_t>(live_hi ? q_hi : 0)) * PF;
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t o1[16], o2[16];
          tc::ld_16x256b_x4(to1 + 32 * ch, o1);
          tc::ld_16x256b_x4(to2 + 32 * ch, o2);
          tc::wait_ld();
#pragma unroll
          for (int gg = 0; gg < 4; ++gg) {
            const int dcol = 32 * ch + 8 * gg + 2 * c4;
            if (live_lo) {
              *reinterpret_cast<float2*>(rec_lo + 4 + dcol) =
                  make_float2(__uint_as_float(o1[4 * gg]), __uint_as_float(o1[4 * gg + 1]));
              *reinterpret_cast<float2*>(rec_lo + 4 + D + dcol) =
                  make_float2(__uint_as_float(o2[4 * gg]), __uint_as_float(o2[4 * gg + 1]));
            }
            if (live_hi) {
              *reinterpret_cast<float2*>(rec_hi + 4 + dcol) =
                  make_float2(__uint_as_float(o1[4 * gg + 2]), __uint_as_float(o1[4 * gg + 3]));
              *reinterpret_cast<float2*>(rec_hi + 4 + D + dcol) =
                  make_float2(__uint_as_float(o2[4 * gg + 2]), __uint_as_float(o2[4 * gg + 3]));
            }
          }
        }
        // O has been read: the next unit's first value MMA may overwrite it
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&o_free[t]));
        if (c4 == 0) {
          if (live_lo) *reinterpret_cast<float4*>(rec_lo) = make_float4(m_lo, l_lo, c_lo, 0.f);
          if (live_hi) *reinterpret_cast<float4*>(rec_hi) = make_float4(m_hi, l_hi, c_hi, 0.f);
        }
      } else {
      const float inv_lo = l_lo > 0.f ? 1.f / l_lo : 0.f;
      const float inv_hi = l_hi > 0.f ? 1.f / l_hi : 0.f;
      const float sb_lo = c_lo * inv_lo, sb_hi = c_hi * inv_hi;  // s_bar = c / l
      const size_t plane = static_cast<size_t>(qplane_of(w, t));
      const size_t lse_row0 = plane * p.lse_stride + w.base;  // lse / sbar index of the sequence's row 0
      // This warp's 16 output rows are staged in shared memory in the 128-byte
      // swizzled layout of the output tensor map and written by one TMA store.
      const uint32_t stage = smem_u32(smem + Cfg::kOffOut) + (t * 4 + wq) * Cfg::kOutWarpBytes;
      if (lane == 0) bulk_wait_read();  // the previous unit's store has read the staging block
      __syncwarp();
      const int r_lo = lane >> 2, r_hi = r_lo + 8;  // rows of this warp's 16
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t o1[16], o2[16];
        tc::ld_16x256b_x4(to1 + 32 * ch, o1);
        tc::ld_16x256b_x4(to2 + 32 * ch, o2);
        tc::wait_ld();
#pragma unroll
        for (int gg = 0; gg < 4; ++gg) {
          const int dcol = 32 * ch + 8 * gg + 2 * c4;
          float r[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float inv = (e & 2) ? inv_hi : inv_lo;
            const float sb = (e & 2) ? sb_hi : sb_lo;
            const float a1 = __uint_as_float(o1[4 * gg + e]) * inv;  // O1 / l
            const float a2 = __uint_as_float(o2[4 * gg + e]) * inv;  // O2 / l
            r[e] = a1 - (a2 - sb * a1);
          }
          const int cb = dcol >> 6, chunk = (dcol & 63) >> 3;
          const uint32_t blk = stage + cb * 2048 + 4 * c4;
          asm volatile("st.shared.u32 [%0], %1;" ::"r"(blk + r_lo * 128 + ((chunk ^ (r_lo & 7)) << 4)),
                       "r"(pack_bf16(r[0], r[1])) : "memory");
          asm volatile("st.shared.u32 [%0], %1;" ::"r"(blk + r_hi * 128 + ((chunk ^ (r_hi & 7)) << 4)),
                       "r"(pack_bf16(r[2], r[3])) : "memory");
        }
      }
      if (!SAVE_AUX) {
        // O has been read: the next unit's first value MMA may overwrite it
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&o_free[t]));
      }
      if (p.lse && c4 == 0) {
        if (q_lo < w.N) p.lse[lse_row0 + q_lo] = l_lo > 0.f ? (m_lo + __log2f(l_lo)) * kLn2 : -INFINITY;
        if (q_hi < w.N) p.lse[lse_row0 + q_hi] = l_hi > 0.f ? (m_hi + __log2f(l_hi)) * kLn2 : -INFINITY;
      }
      fence_proxy_async_smem();
      __syncwarp();
      const int row0 = q0 + 16 * wq;
      // Packed sequences: a 16-row group that runs past its sequence would
      // overwrite the next sequence's rows, so its live rows are copied out of
      // the staging block with plain stores instead of the TMA store.
      const bool partial = p.cu_seqlens != nullptr && row0 < w.N && row0 + 16 > w.N;
      auto copy_rows = [&](__nv_bfloat16* dst) {
        const int nrows = w.N - row0;
        for (int i = lane; i < nrows * Cfg::kCB * 8; i += 32) {
          const int rr = i / (Cfg::kCB * 8), cb = (i / 8) % Cfg::kCB, c = i % 8;
          uint4 v;
          asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                       : "r"(stage + cb * 2048 + rr * 128 + ((c ^ (rr & 7)) << 4)));
          const size_t tok = static_cast<size_t>(w.base + row0 + rr);
          *reinterpret_cast<uint4*>(dst + (tok * p.Hq + head_of(w, t)) * D + cb * 64 + c * 8) = v;
        }
        __syncwarp();
      };
      if (partial) {
        copy_rows(p.out);
      } else if (lane == 0 && row0 < w.N) {
#pragma unroll
        for (int cb = 0; cb < Cfg::kCB; ++cb)
          tma_store_3d(&omap, stage + cb * 2048, cb * 64, w.base + row0, static_cast<int>(plane));
        bulk_commit();
      }
      if (SAVE_AUX) {
        // Training forward: keep s_bar = c / l and o_bar = O1 / l (the softmax
        // output) for the backward.  o_bar goes through the same staging
        // block once the output store has read it.
        if (p.sbar && c4 == 0) {
          if (q_lo < w.N) p.sbar[lse_row0 + q_lo] = sb_lo;
          if (q_hi < w.N) p.sbar[lse_row0 + q_hi] = sb_hi;
        }
        if (lane == 0) bulk_wait_read();
        __syncwarp();
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t o1[16];
          tc::ld_16x256b_x4(to1 + 32 * ch, o1);
          tc::wait_ld();
#pragma unroll
          for (int gg = 0; gg < 4; ++gg) {
            const int dcol = 32 * ch + 8 * gg + 2 * c4;
            const int cb = dcol >> 6, chunk = (dcol & 63) >> 3;
            const uint32_t blk = stage + cb * 2048 + 4 * c4;
            asm volatile("st.shared.u32 [%0], %1;" ::"r"(blk + r_lo * 128 + ((chunk ^ (r_lo & 7)) << 4)),
                         "r"(pack_bf16(__uint_as_float(o1[4 * gg]) * inv_lo, __uint_as_float(o1[4 * gg + 1]) * inv_lo))
                         : "memory");
            asm volatile("st.shared.u32 [%0], %1;" ::"r"(blk + r_hi * 128 + ((chunk ^ (r_hi & 7)) << 4)),
                         "r"(pack_bf16(__uint_as_float(o1[4 * gg + 2]) * inv_hi, __uint_as_float(o1[4 * gg + 3]) * inv_hi))
                         : "memory");
          }
        }
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&o_free[t]));
        fence_proxy_async_smem();
        __syncwarp();
        if (partial) {
          copy_rows(p.obar);
        } else if (lane == 0 && row0 < w.N) {
#pragma unroll
          for (int cb = 0; cb < Cfg::kCB; ++cb)
            tma_store_3d(&amap, stage + cb * 2048, cb * 64, w.base + row0, static_cast<int>(plane));
          bulk_commit();
        }
      }
      }  // output epilogue
      kv += w.nkv;
      ++n_unit;
    }
    if (lane == 0) bulk_wait_all();  // output stores complete before exit
    tc::fence_before_sync();
    asm volatile("bar.sync 1, %0;" ::"n"(kFwdThreads) : "memory");  // every role is done
  }
}

}  // namespace plx
