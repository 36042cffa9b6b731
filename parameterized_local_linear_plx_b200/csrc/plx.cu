// plx.cu -- the C ABI of libplx.so (declared in include/plx.h): argument
// validation, TMA descriptor set-up, split selection and kernel launches.
// No device or host memory is allocated here; the caller owns every buffer.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <algorithm>
#include <mutex>

#include "../../include/plx.h"
#include "plx_append.cuh"
#include "plx_bwd.cuh"
#include "plx_decode.cuh"
#include "plx_fwd.cuh"
#include "plx_proj.cuh"

namespace {

constexpr int kMaxDevices = 64;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---------------------------------------------------------------- device checks
int g_arch_ok[kMaxDevices];  // 0 unknown, 1 ok, -1 not sm_100
int g_sm_count[kMaxDevices];
std::mutex g_mu;

int check_arch(int* dev_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PLX_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return PLX_ERR_CUDA;
  *dev_out = dev;
  if (g_arch_ok[dev] == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return PLX_ERR_CUDA;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
      return PLX_ERR_CUDA;
    g_sm_count[dev] = sms;
    g_arch_ok[dev] = (major == 10 && minor == 0) ? 1 : -1;
  }
  return g_arch_ok[dev] == 1 ? PLX_OK : PLX_ERR_ARCH;
}

// ---------------------------------------------------------------- tensor maps
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int get_encoder() {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_encode) return PLX_OK;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q{};
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || fn == nullptr)
    return PLX_ERR_CUDA;
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return PLX_OK;
}

// A bf16 tensor [planes, rows, D] (D contiguous) as a 3-D TMA map with a
// box of {64 elements, box_rows, 1} and 128-byte swizzle.  Loads past `rows`
// (inside a plane) are zero-filled, so ragged tails never read a neighbour.
// Encoded maps are cached per (base, D, rows, planes, box_rows): a decode
// step at a steady shape re-encodes nothing (the encode is host work on the
// critical path of a small call).  A map holds only the address, extents and
// strides, so a cached entry stays valid for any buffer at that address.
struct MapKey {
  const void* base;
  long long rows, planes;
  int D, box_rows;
};
constexpr int kMapCache = 64;
MapKey g_map_keys[kMapCache];
CUtensorMap g_map_vals[kMapCache];
int g_map_next = 0;
std::mutex g_map_mu;

int encode_map_3d(CUtensorMap* map, const void* base, int D, long long rows, long long planes, int box_rows);

int make_map_3d(CUtensorMap* map, const void* base, int D, long long rows, long long planes, int box_rows) {
  {
    std::lock_guard<std::mutex> lk(g_map_mu);
    for (int i = 0; i < kMapCache; ++i) {
      const MapKey& k = g_map_keys[i];
      if (k.base == base && k.base != nullptr && k.rows == rows && k.planes == planes && k.D == D &&
          k.box_rows == box_rows) {
        *map = g_map_vals[i];
        return PLX_OK;
      }
    }
  }
  const int rc = encode_map_3d(map, base, D, rows, planes, box_rows);
  if (rc == PLX_OK) {
    std::lock_guard<std::mutex> lk(g_map_mu);
    g_map_keys[g_map_next] = MapKey{base, rows, planes, D, box_rows};
    g_map_vals[g_map_next] = *map;
    g_map_next = (g_map_next + 1) % kMapCache;
  }
  return rc;
}

int encode_map_3d(CUtensorMap* map, const void* base, int D, long long rows, long long planes, int box_rows) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(planes)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2u,
                           static_cast<cuuint64_t>(rows) * static_cast<cuuint64_t>(D) * 2u};
  cuuint32_t box[3] = {64u, static_cast<cuuint32_t>(box_rows), 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult rc = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return rc == CUDA_SUCCESS ? PLX_OK : PLX_ERR_CUDA;
}

// A token-major bf16 tensor [rows, planes, D] (packed sequences: a row is a
// token, a plane a head) as the same 3-D view {D, rows, planes}: the row
// stride is planes * D elements and the plane stride D elements.  Loads past
// the last row are zero-filled.
int make_map_3d_tokens(CUtensorMap* map, const void* base, int D, long long rows, long long planes, int box_rows) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(planes)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(planes) * static_cast<cuuint64_t>(D) * 2u,
                           static_cast<cuuint64_t>(D) * 2u};
  cuuint32_t box[3] = {64u, static_cast<cuuint32_t>(box_rows), 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult rc = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return rc == CUDA_SUCCESS ? PLX_OK : PLX_ERR_CUDA;
}

// A row-major bf16 matrix [rows, cols] as a 2-D TMA map with a box of
// {64 columns, box_rows rows} and 128-byte swizzle; loads past either extent
// are zero-filled.
int make_map_2d(CUtensorMap* map, const void* base, long long cols, long long rows, int box_rows) {
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2u};
  cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult rc = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return rc == CUDA_SUCCESS ? PLX_OK : PLX_ERR_CUDA;
}

// Opt a kernel into more than 48 KB of dynamic shared memory, once per device.
template <typename K>
int ensure_smem(K kernel, int bytes, bool* done) {
  if (*done) return PLX_OK;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return PLX_ERR_CUDA;
  *done = true;
  return PLX_OK;
}

// ---------------------------------------------------------------- decode
// The decode split kernel runs P persistent CTAs (two per SM by default) over
// the key tiles of the whole batch; its scratch holds two partial-state slots
// per CTA (rows_per_slot rows each) and one int4 per CTA for the combine.
size_t align256(size_t n) { return (n + 255) / 256 * 256; }

int sm_count_or_default() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) == cudaSuccess &&
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && sms > 0)
    return sms;
  return 148;  // B200
}

// The balanced plan's default CTA count: one per SM when segments are long
// (fewer, longer ranges: fewer partial states to merge), two per SM for
// short segments (at most 256 keys), whose cost is per segment rather than
// per key.  Both measured on every shape the plan serves.
int decode_ctas(int num_splits, int S_max) {
  if (num_splits > 0) return num_splits;
  return (S_max <= 256 ? 2 : 1) * sm_count_or_default();
}

int rows_per_slot(int Hq, int Hkv) { return std::min(Hq / Hkv, 8); }

size_t decode_scratch_bytes(int Hq, int Hkv, int d, int P) {
  return align256(static_cast<size_t>(2) * P * rows_per_slot(Hq, Hkv) * (2 * d + 4) * sizeof(float));
}

// Two plans share the decode kernel.  The balanced plan (persistent CTAs over
// equal ranges of the batch's tile list) wins when the batch has few (b, kv
// head) segments, or short ones; with many long segments the chunked plan
// (one CTA per chunk of a segment, like a split-KV grid, several waves)
// streams the cache faster.  Measured crossover: 128 segments or more, of
// more than 256 keys.
constexpr long long kChunkedMinSegments = 128;
constexpr int kChunkedMinKeys = 256;
// The segment plan (one warp streams each whole segment, one kernel, no
// partial states) for contiguous caches whose segments are all short.
constexpr int kSegMaxKeys = 256;

struct DecodePlan {
  bool chunked;
  bool seg;         // segment plan
  bool seg_many;    // segment plan, the 8-warp shape with 16-key stages
  int P;            // CTAs of the decode kernel
  int splits;       // chunked: parts per segment
  int chunk_tiles;  // chunked: tiles per part
  size_t ws_bytes;  // workspace the plan needs
};

DecodePlan plan_decode(int B, int Hq, int Hkv, int S_max, int d, int num_splits, bool records, bool paged) {
  DecodePlan pl{};
  const int n_hg = (Hq / Hkv + 7) / 8;
  const long long segs = static_cast<long long>(B) * Hkv * n_hg;
  if (num_splits == 0 && !paged && S_max <= kSegMaxKeys && segs <= 0x7fffffffLL) {
    // one CTA per SM (fewer when there are fewer segments); the 8-warp shape
    // once the segments outnumber the 4-warp shape's warps and are at most
    // 128 keys long (measured: 1.25x faster at 2048-16384 segments of <= 128
    // keys, equal at 512, 5% slower for 4096 segments of 128-256 keys)
    const int sms = sm_count_or_default();
    pl.seg = true;
    pl.seg_many = segs > static_cast<long long>(plx::kSegFewWarps) * sms && S_max <= 128;
    pl.P = static_cast<int>(std::min<long long>(segs, sms));
    pl.ws_bytes = 0;
    return pl;
  }
  if (num_splits == 0 && !records && segs >= kChunkedMinSegments && S_max > kChunkedMinKeys && B <= 65535 &&
      static_cast<long long>(Hkv) * n_hg <= 65535) {
    // about four waves of two CTAs per SM, chunks of at least 128 keys
    const long long target = 4LL * 2 * sm_count_or_default();
    long long sp = (target + segs - 1) / segs;
    const long long max_sp = (S_max + 127) / 128;
    sp = std::max(1LL, std::min(sp, max_sp));
    const int keys = static_cast<int>((S_max + sp - 1) / sp);
    pl.chunked = true;
    pl.chunk_tiles = (keys + plx::kDecTileKeys - 1) / plx::kDecTileKeys;
    pl.splits = (S_max + pl.chunk_tiles * plx::kDecTileKeys - 1) / (pl.chunk_tiles * plx::kDecTileKeys);
    pl.P = static_cast<int>(std::min<long long>(segs * pl.splits, 0x7fffffffLL));
    pl.ws_bytes = pl.splits > 1 ? align256(static_cast<size_t>(B) * Hq * pl.splits * (2 * d + 4) * sizeof(float)) : 0;
    return pl;
  }
  pl.chunked = false;
  pl.P = decode_ctas(num_splits, S_max);
  pl.ws_bytes = decode_scratch_bytes(Hq, Hkv, d, pl.P);
  return pl;
}

template <int D, bool HAS_R, bool PAGED>
int launch_decode(const CUtensorMap& km, const CUtensorMap& vm, const CUtensorMap& kt, const CUtensorMap& vt,
                  const CUtensorMap* k32, const CUtensorMap* v32, const plx::DecodeParams& p,
                  const DecodePlan& plan, cudaStream_t st) {
  using Cfg = plx::DecodeCfg<D>;
  static bool done[kMaxDevices], done_chunk[kMaxDevices], done_seg[kMaxDevices], done_seg_many[kMaxDevices];
  int dev = 0;
  cudaGetDevice(&dev);
  const int P = plan.P;
  if constexpr (!PAGED) {
    if (plan.seg) {
      // k32 / v32: maps with the shape's stage height (32 or 16 keys)
      if (plan.seg_many) {
        using SC = plx::SegCfg<D, plx::kSegManyWarps, plx::kSegManyKeys>;
        auto kern = plx::plx_decode_seg_kernel<D, HAS_R, plx::kSegManyWarps, plx::kSegManyKeys>;
        if (ensure_smem(kern, SC::kSmemBytes, &done_seg_many[dev]) != PLX_OK) return PLX_ERR_CUDA;
        kern<<<static_cast<unsigned>(P), SC::kThreads, SC::kSmemBytes, st>>>(*k32, *v32, kt, vt, p);
      } else {
        using SC = plx::SegCfg<D, plx::kSegFewWarps, plx::kSegFewKeys>;
        auto kern = plx::plx_decode_seg_kernel<D, HAS_R, plx::kSegFewWarps, plx::kSegFewKeys>;
        if (ensure_smem(kern, SC::kSmemBytes, &done_seg[dev]) != PLX_OK) return PLX_ERR_CUDA;
        kern<<<static_cast<unsigned>(P), SC::kThreads, SC::kSmemBytes, st>>>(*k32, *v32, kt, vt, p);
      }
      return cudaGetLastError() == cudaSuccess ? PLX_OK : PLX_ERR_CUDA;
    }
  }
  if (p.chunk_tiles > 0) {
    auto kern = plx::plx_decode_chunk_kernel<D, HAS_R, PAGED>;
    if (ensure_smem(kern, Cfg::kChunkSmemBytes, &done_chunk[dev]) != PLX_OK) return PLX_ERR_CUDA;
    const dim3 grid(static_cast<unsigned>(p.splits), static_cast<unsigned>(p.Hkv * p.n_hgroups),
                    static_cast<unsigned>(p.B));
    kern<<<grid, plx::kDecThreads, Cfg::kChunkSmemBytes, st>>>(km, vm, kt, vt, p);
    if (cudaGetLastError() != cudaSuccess) return PLX_ERR_CUDA;
    if (p.splits == 1) return PLX_OK;  // every segment was finished whole
  } else {
    auto kern = plx::plx_decode_split_kernel<D, HAS_R, PAGED>;
    if (ensure_smem(kern, Cfg::kSmemBytes, &done[dev]) != PLX_OK) return PLX_ERR_CUDA;
    kern<<<static_cast<unsigned>(P), plx::kDecThreads, Cfg::kSmemBytes, st>>>(km, vm, kt, vt, p);
    if (cudaGetLastError() != cudaSuccess) return PLX_ERR_CUDA;
  }
  // programmatic dependent launch: the second kernel's CTAs are scheduled
  // while the decode grid runs, and griddepcontrol.wait inside it orders its
  // reads after that grid's completion
  cudaLaunchConfig_t cfg{};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  if (p.chunk_tiles > 0) {
    // the parts of every row: [B * Hq rows, splits, 2D + 4] merged one warp per row
    const long long rows = static_cast<long long>(p.B) * p.Hq;
    const long long threads = rows * (D / 4);
    cfg.gridDim = dim3(static_cast<unsigned>((threads + 255) / 256));
    cfg.blockDim = dim3(256);
    const long long rf = 2 * D + 4;
    if (cudaLaunchKernelEx(&cfg, plx::plx_record_merge_kernel<D>, static_cast<const float*>(p.ws), p.splits, rows,
                           p.out, p.lse, rf, rf * p.splits) != cudaSuccess)
      return PLX_ERR_CUDA;
    return PLX_OK;
  }
  // balanced plan: one combine CTA per SM (each can be resident beside the
  // split CTAs), at most a few split CTAs' jobs each
  const int sms = sm_count_or_default();
  const int cgrid = std::max(std::min(P, sms), (P + 3) / 4);
  cfg.gridDim = dim3(static_cast<unsigned>(cgrid));
  cfg.blockDim = dim3(plx::kDecCombineThreads);
  if (cudaLaunchKernelEx(&cfg, plx::plx_decode_combine_kernel<D>, p, P) != cudaSuccess) return PLX_ERR_CUDA;
  return PLX_OK;
}

template <int D, bool HAS_R, int MODE>
int launch_fwd(const CUtensorMap& qm, const CUtensorMap& rm, const CUtensorMap& km, const CUtensorMap& vm,
               const CUtensorMap& om, const CUtensorMap& am, const plx::FwdParams& p, unsigned grid,
               cudaStream_t st) {
  using Cfg = plx::FwdCfg<D>;
  static bool done[kMaxDevices];
  int dev = 0;
  cudaGetDevice(&dev);
  auto kern = plx::plx_fwd_kernel<D, HAS_R, MODE>;
  if (ensure_smem(kern, Cfg::kSmemBytes, &done[dev]) != PLX_OK) return PLX_ERR_CUDA;
  kern<<<grid, plx::kFwdThreads, Cfg::kSmemBytes, st>>>(qm, rm, km, vm, om, am, p);
  return cudaGetLastError() == cudaSuccess ? PLX_OK : PLX_ERR_CUDA;
}

template <int D, bool HAS_R>
int launch_bwd(const CUtensorMap& qm, const CUtensorMap& rm, const CUtensorMap& om, const CUtensorMap& km,
               const CUtensorMap& vm, const CUtensorMap& kmq, const CUtensorMap& vmq, const plx::BwdParams& p, const void* dout, const void* out,
               const void* obar, float* gbar, float* dd, cudaStream_t st) {
  using QCfg = plx::BwdQCfg<D>;
  using KVCfg = plx::BwdKVCfg<D>;
  static bool done_q[kMaxDevices], done_kv[kMaxDevices];
  int dev = 0;
  cudaGetDevice(&dev);
  const long long rows = static_cast<long long>(p.B) * p.Hq * p.N;
  plx::plx_bwd_pre_kernel<D><<<static_cast<unsigned>((rows + 7) / 8), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(dout), static_cast<const __nv_bfloat16*>(out),
      static_cast<const __nv_bfloat16*>(obar), p.sbar, gbar, dd, rows);
  if (cudaGetLastError() != cudaSuccess) return PLX_ERR_CUDA;
  auto kq = plx::plx_bwd_q_kernel<D, HAS_R>;
  if (ensure_smem(kq, QCfg::kSmemBytes, &done_q[dev]) != PLX_OK) return PLX_ERR_CUDA;
  kq<<<static_cast<unsigned>(p.B * p.Hq * p.n_qtiles), plx::kBwdThreads, QCfg::kSmemBytes, st>>>(qm, rm, om, kmq, vmq, p);
  if (cudaGetLastError() != cudaSuccess) return PLX_ERR_CUDA;
  auto kkv = plx::plx_bwd_kv_kernel<D, HAS_R>;
  if (ensure_smem(kkv, KVCfg::kSmemBytes, &done_kv[dev]) != PLX_OK) return PLX_ERR_CUDA;
  kkv<<<static_cast<unsigned>(p.B * p.Hkv * p.n_ktiles), plx::kBwdThreads, KVCfg::kSmemBytes, st>>>(qm, rm, om, km, vm, p);
  return cudaGetLastError() == cudaSuccess ? PLX_OK : PLX_ERR_CUDA;
}

size_t bwd_workspace_bytes(int B, int Hq, int N) {
  const size_t rows = static_cast<size_t>(B) * Hq * N;
  return 2 * ((rows * sizeof(float) + 255) / 256 * 256);
}

}  // namespace

extern "C" {

int plx_version(void) { return 100; }

const char* plx_status_string(int status) {
  switch (status) {
    case PLX_OK: return "PLX_OK";
    case PLX_ERR_NULL: return "PLX_ERR_NULL: a required pointer is NULL";
    case PLX_ERR_SHAPE: return "PLX_ERR_SHAPE: a size is out of range";
    case PLX_ERR_HEADDIM: return "PLX_ERR_HEADDIM: head dim must be 64 or 128";
    case PLX_ERR_GQA: return "PLX_ERR_GQA: Hq must be a multiple of Hkv";
    case PLX_ERR_ALIGN: return "PLX_ERR_ALIGN: pointers must be 16-byte aligned";
    case PLX_ERR_WORKSPACE: return "PLX_ERR_WORKSPACE: workspace missing or too small";
    case PLX_ERR_CUDA: return "PLX_ERR_CUDA: a CUDA call failed";
    case PLX_ERR_DEVICE_TIMEOUT: return "PLX_ERR_DEVICE_TIMEOUT: a kernel gave up a bounded wait";
    case PLX_ERR_ARCH: return "PLX_ERR_ARCH: the current device is not sm_100";
    default: return "PLX: unknown status";
  }
}

}  // extern "C"

namespace {

// plx_fwd and plx_fwd_train: obar / sbar non-NULL selects the training kernel.
// cu_seqlens non-NULL: packed sequences (token-major [total, H, d]), N = the
// longest sequence.
int fwd_common(const void* q, const void* k, const void* v, const void* r, void* out, float* lse,
               void* obar, float* sbar, int B, int Hq, int Hkv, int N, int d, int causal, float scale,
               void* stream, const int* cu_seqlens = nullptr, int total = 0, float* partial = nullptr) {
  if (!q || !k || !v || (!out && !partial)) return PLX_ERR_NULL;
  if (B < 1 || Hq < 1 || Hkv < 1 || N < 1) return PLX_ERR_SHAPE;
  if (d != 64 && d != 128) return PLX_ERR_HEADDIM;
  if (Hq % Hkv) return PLX_ERR_GQA;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || (r && !aligned16(r)) || (out && !aligned16(out)) ||
      (partial && !aligned16(partial)) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) || (obar && !aligned16(obar)) ||
      (sbar && (reinterpret_cast<uintptr_t>(sbar) & 3u)) || (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u))
    return PLX_ERR_ALIGN;
  const bool packed = cu_seqlens != nullptr;
  if (packed && total < 1) return PLX_ERR_SHAPE;
  const bool train = obar != nullptr;
  const int G = Hq / Hkv;
  const int pair_heads = (G % 2 == 0) ? 1 : 0;
  const int n_pairs = pair_heads ? Hq / 2 : Hq;
  const int n_qblocks = pair_heads ? (N + plx::kFwdBM - 1) / plx::kFwdBM : (N + 2 * plx::kFwdBM - 1) / (2 * plx::kFwdBM);
  const long long grid = static_cast<long long>(B) * n_pairs * n_qblocks;
  if (grid > 0x7fffffffLL) return PLX_ERR_SHAPE;
  int dev = 0;
  int rc = check_arch(&dev);
  if (rc != PLX_OK) return rc;
  if ((rc = get_encoder()) != PLX_OK) return rc;

  CUtensorMap qm, rm, km, vm, om, am;
  const long long pq = static_cast<long long>(B) * Hq, pkv = static_cast<long long>(B) * Hkv;
  // fixed length: [planes = B * H, rows = N]; packed: [planes = H, rows = total] over token-major storage
  auto map_q = [&](CUtensorMap* m, const void* base) {
    return packed ? make_map_3d_tokens(m, base, d, total, Hq, 16) : make_map_3d(m, base, d, N, pq, 16);
  };
  auto map_kv = [&](CUtensorMap* m, const void* base) {
    return packed ? make_map_3d_tokens(m, base, d, total, Hkv, plx::kFwdBN) : make_map_3d(m, base, d, N, pkv, plx::kFwdBN);
  };
  if (map_q(&qm, q) != PLX_OK || map_kv(&km, k) != PLX_OK || map_kv(&vm, v) != PLX_OK)
    return PLX_ERR_CUDA;
  if (out) {
    if (map_q(&om, out) != PLX_OK) return PLX_ERR_CUDA;
  } else {
    om = qm;  // unused: the partial-state forward writes no output tile
  }
  if (r) {
    if (map_q(&rm, r) != PLX_OK) return PLX_ERR_CUDA;
  } else {
    rm = qm;  // unused
  }
  if (train) {
    if (map_q(&am, obar) != PLX_OK) return PLX_ERR_CUDA;
  } else {
    am = om;  // unused
  }
  plx::FwdParams p;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.sbar = sbar;
  p.obar = static_cast<__nv_bfloat16*>(obar);
  p.cu_seqlens = cu_seqlens;
  p.total = total;
  p.lse_stride = packed ? total : N;
  p.partial = partial;
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.N = N; p.G = G;
  p.pair_heads = pair_heads; p.n_pairs = n_pairs; p.n_qblocks = n_qblocks;
  p.num_units = static_cast<int>(grid);
  p.causal = causal ? 1 : 0;
  p.scale_log2 = scale * plx::kLog2e;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // persistent: one CTA per SM (the kernel's shared memory allows no more)
  const unsigned g = static_cast<unsigned>(std::min<long long>(grid, g_sm_count[dev]));
  if (partial) {
    constexpr int M = plx::kFwdModePartial;
    if (d == 128)
      return r ? launch_fwd<128, true, M>(qm, rm, km, vm, om, am, p, g, st)
               : launch_fwd<128, false, M>(qm, rm, km, vm, om, am, p, g, st);
    return r ? launch_fwd<64, true, M>(qm, rm, km, vm, om, am, p, g, st)
             : launch_fwd<64, false, M>(qm, rm, km, vm, om, am, p, g, st);
  }
  if (train) {
    constexpr int M = plx::kFwdModeTrain;
    if (d == 128)
      return r ? launch_fwd<128, true, M>(qm, rm, km, vm, om, am, p, g, st)
               : launch_fwd<128, false, M>(qm, rm, km, vm, om, am, p, g, st);
    return r ? launch_fwd<64, true, M>(qm, rm, km, vm, om, am, p, g, st)
             : launch_fwd<64, false, M>(qm, rm, km, vm, om, am, p, g, st);
  }
  constexpr int M = plx::kFwdModeOut;
  if (d == 128)
    return r ? launch_fwd<128, true, M>(qm, rm, km, vm, om, am, p, g, st)
             : launch_fwd<128, false, M>(qm, rm, km, vm, om, am, p, g, st);
  return r ? launch_fwd<64, true, M>(qm, rm, km, vm, om, am, p, g, st)
           : launch_fwd<64, false, M>(qm, rm, km, vm, om, am, p, g, st);
}

}  // namespace

extern "C" {

int plx_fwd(const void* q, const void* k, const void* v, const void* r, void* out, float* lse, int B,
            int Hq, int Hkv, int N, int d, int causal, float scale, void* stream) {
  return fwd_common(q, k, v, r, out, lse, nullptr, nullptr, B, Hq, Hkv, N, d, causal, scale, stream);
}

int plx_fwd_train(const void* q, const void* k, const void* v, const void* r, void* out, float* lse,
                  void* obar, float* sbar, int B, int Hq, int Hkv, int N, int d, int causal, float scale,
                  void* stream) {
  if (!lse || !obar || (r && !sbar)) return PLX_ERR_NULL;
  return fwd_common(q, k, v, r, out, lse, obar, sbar, B, Hq, Hkv, N, d, causal, scale, stream);
}

int plx_fwd_varlen(const void* q, const void* k, const void* v, const void* r, void* out, float* lse,
                   const int32_t* cu_seqlens, int B, int Hq, int Hkv, int total, int max_seqlen, int d, int causal,
                   float scale, void* stream) {
  if (!cu_seqlens) return PLX_ERR_NULL;
  return fwd_common(q, k, v, r, out, lse, nullptr, nullptr, B, Hq, Hkv, max_seqlen, d, causal, scale, stream,
                    cu_seqlens, total);
}

size_t plx_fwd_partial_size(int B, int Hq, int N, int d) {
  if (B < 1 || Hq < 1 || N < 1 || (d != 64 && d != 128)) return 0;
  return static_cast<size_t>(B) * Hq * N * (2 * d + 4) * sizeof(float);
}

int plx_fwd_partial(const void* q, const void* k, const void* v, const void* r, float* partial, size_t partial_bytes,
                    int B, int Hq, int Hkv, int N, int d, int causal, float scale, void* stream) {
  if (!partial) return PLX_ERR_NULL;
  const size_t need = plx_fwd_partial_size(B, Hq, N, d);
  if (need != 0 && partial_bytes < need) return PLX_ERR_WORKSPACE;  // bad shapes: fwd_common reports them
  return fwd_common(q, k, v, r, nullptr, nullptr, nullptr, nullptr, B, Hq, Hkv, N, d, causal, scale, stream, nullptr,
                    0, partial);
}

int plx_decode_paged(const void* q, const void* r, const void* kpool, const void* vpool,
                     const int32_t* block_table, const int32_t* seqlens, void* out, float* lse, int B, int Hq,
                     int Hkv, int num_pages, int page_size, int max_pages, int d, float scale, int num_splits,
                     void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !kpool || !vpool || !block_table || !seqlens || !out) return PLX_ERR_NULL;
  if (B < 1 || Hq < 1 || Hkv < 1 || num_pages < 1 || max_pages < 1 || num_splits < 0) return PLX_ERR_SHAPE;
  if (page_size < 16 || page_size > 4096 || (page_size & (page_size - 1))) return PLX_ERR_SHAPE;
  if (static_cast<long long>(max_pages) * page_size > 0x7fffffffLL ||
      static_cast<long long>(num_pages) * Hkv > 0x7fffffffLL)
    return PLX_ERR_SHAPE;
  if (d != 64 && d != 128) return PLX_ERR_HEADDIM;
  if (Hq % Hkv) return PLX_ERR_GQA;
  if (!aligned16(q) || (r && !aligned16(r)) || !aligned16(kpool) || !aligned16(vpool) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(seqlens) & 3u) || (reinterpret_cast<uintptr_t>(block_table) & 3u) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return PLX_ERR_ALIGN;
  const int S_max = max_pages * page_size;
  const DecodePlan plan = plan_decode(B, Hq, Hkv, S_max, d, num_splits, false, true);
  if (plan.ws_bytes > 0 && (!workspace || workspace_bytes < plan.ws_bytes)) return PLX_ERR_WORKSPACE;
  if (plan.ws_bytes > 0 && !aligned16(workspace)) return PLX_ERR_ALIGN;
  const int G = Hq / Hkv;
  const int n_hg = (G + 7) / 8;
  if (static_cast<long long>(B) * Hkv * n_hg * ((S_max + plx::kDecTileKeys - 1) / plx::kDecTileKeys) > 0x7fffffffLL)
    return PLX_ERR_SHAPE;
  int dev = 0;
  int rc = check_arch(&dev);
  if (rc != PLX_OK) return rc;
  if ((rc = get_encoder()) != PLX_OK) return rc;

  // the pools as [num_pages * Hkv planes, page_size rows, d]; one box = one page part
  const int box_rows = page_size < plx::kDecTileKeys ? page_size : plx::kDecTileKeys;
  CUtensorMap km, vm;
  const long long planes = static_cast<long long>(num_pages) * Hkv;
  if (make_map_3d(&km, kpool, d, page_size, planes, box_rows) != PLX_OK ||
      make_map_3d(&vm, vpool, d, page_size, planes, box_rows) != PLX_OK)
    return PLX_ERR_CUDA;

  plx::DecodeParams p{};
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.r = static_cast<const __nv_bfloat16*>(r);
  p.seqlens = seqlens;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.block_table = block_table;
  p.num_pages = num_pages;
  p.max_pages = max_pages;
  p.page_size = page_size;
  int shift = 0;
  while ((1 << shift) < page_size) ++shift;
  p.page_shift = shift;
  p.box_rows = box_rows;
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.S_max = S_max; p.G = G; p.n_hgroups = n_hg;
  p.rps = rows_per_slot(Hq, Hkv);
  p.ws = static_cast<float*>(workspace);
  p.chunk_tiles = plan.chunked ? plan.chunk_tiles : 0;
  p.splits = plan.chunked ? plan.splits : 0;
  p.scale_log2 = scale * plx::kLog2e;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // (the partial-tile maps are for contiguous caches; page parts carry their own box)
  if (d == 128)
    return r ? launch_decode<128, true, true>(km, vm, km, vm, nullptr, nullptr, p, plan, st)
             : launch_decode<128, false, true>(km, vm, km, vm, nullptr, nullptr, p, plan, st);
  return r ? launch_decode<64, true, true>(km, vm, km, vm, nullptr, nullptr, p, plan, st)
           : launch_decode<64, false, true>(km, vm, km, vm, nullptr, nullptr, p, plan, st);
}

}  // extern "C"

namespace {

int append_common(const void* knew, const void* vnew, void* kc, void* vc, int32_t* seqlens,
                  const int32_t* block_table, int B, int Hkv, int S_max, int num_pages, int page_size,
                  int max_pages, int d, int advance, void* stream) {
  if (!knew || !vnew || !kc || !vc || !seqlens) return PLX_ERR_NULL;
  if (d != 64 && d != 128) return PLX_ERR_HEADDIM;
  if (!aligned16(knew) || !aligned16(vnew) || !aligned16(kc) || !aligned16(vc) ||
      (reinterpret_cast<uintptr_t>(seqlens) & 3u) || (reinterpret_cast<uintptr_t>(block_table) & 3u))
    return PLX_ERR_ALIGN;
  int dev = 0;
  int rc = check_arch(&dev);
  if (rc != PLX_OK) return rc;
  plx::AppendParams p{};
  p.knew = static_cast<const __nv_bfloat16*>(knew);
  p.vnew = static_cast<const __nv_bfloat16*>(vnew);
  p.kcache = static_cast<__nv_bfloat16*>(kc);
  p.vcache = static_cast<__nv_bfloat16*>(vc);
  p.seqlens = seqlens;
  p.block_table = block_table;
  p.B = B; p.Hkv = Hkv; p.S_max = S_max;
  p.num_pages = num_pages; p.page_size = page_size; p.max_pages = max_pages;
  int shift = 0;
  while (page_size > 0 && (1 << shift) < page_size) ++shift;
  p.page_shift = shift;
  p.advance = advance ? 1 : 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const unsigned grid = static_cast<unsigned>((B + 7) / 8);
  if (d == 128)
    plx::plx_kv_append_kernel<128><<<grid, 256, 0, st>>>(p);
  else
    plx::plx_kv_append_kernel<64><<<grid, 256, 0, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? PLX_OK : PLX_ERR_CUDA;
}

}  // namespace

extern "C" {

int plx_kv_append(const void* knew, const void* vnew, void* kcache, void* vcache, int32_t* seqlens, int B,
                  int Hkv, int S_max, int d, int advance, void* stream) {
  if (B < 1 || Hkv < 1 || S_max < 1) return PLX_ERR_SHAPE;
  return append_common(knew, vnew, kcache, vcache, seqlens, nullptr, B, Hkv, S_max, 0, 0, 0, d, advance, stream);
}

int plx_kv_append_paged(const void* knew, const void* vnew, void* kpool, void* vpool, const int32_t* block_table,
                        int32_t* seqlens, int B, int Hkv, int num_pages, int page_size, int max_pages, int d,
                        int advance, void* stream) {
  if (!block_table) return PLX_ERR_NULL;
  if (B < 1 || Hkv < 1 || num_pages < 1 || max_pages < 1) return PLX_ERR_SHAPE;
  if (page_size < 16 || page_size > 4096 || (page_size & (page_size - 1))) return PLX_ERR_SHAPE;
  if (static_cast<long long>(max_pages) * page_size > 0x7fffffffLL) return PLX_ERR_SHAPE;
  return append_common(knew, vnew, kpool, vpool, seqlens, block_table, B, Hkv, 0, num_pages, page_size, max_pages,
                       d, advance, stream);
}

size_t plx_bwd_workspace_size(int B, int Hq, int Hkv, int N, int d) {
  if (B < 1 || Hq < 1 || Hkv < 1 || N < 1 || Hq % Hkv || (d != 64 && d != 128)) return 0;
  return bwd_workspace_bytes(B, Hq, N);
}

int plx_bwd(const void* q, const void* k, const void* v, const void* r, const void* out, const void* dout,
            const float* lse, const void* obar, const float* sbar, void* dq, void* dk, void* dv, void* dr,
            int B, int Hq, int Hkv, int N, int d, int causal, float scale, void* workspace,
            size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !out || !dout || !lse || !obar || !dq || !dk || !dv || (r && !sbar)) return PLX_ERR_NULL;
  if (B < 1 || Hq < 1 || Hkv < 1 || N < 1) return PLX_ERR_SHAPE;
  if (d != 64 && d != 128) return PLX_ERR_HEADDIM;
  if (Hq % Hkv) return PLX_ERR_GQA;
  const void* p16[] = {q, k, v, r, out, dout, obar, dq, dk, dv, dr, workspace};
  for (const void* ptr : p16)
    if (ptr && !aligned16(ptr)) return PLX_ERR_ALIGN;
  if ((reinterpret_cast<uintptr_t>(lse) & 3u) || (sbar && (reinterpret_cast<uintptr_t>(sbar) & 3u)))
    return PLX_ERR_ALIGN;
  const size_t need = bwd_workspace_bytes(B, Hq, N);
  if (!workspace || workspace_bytes < need) return PLX_ERR_WORKSPACE;
  const int n_qtiles = (N + plx::kBwdBM - 1) / plx::kBwdBM;
  const int n_ktiles = (N + plx::kBwdBN - 1) / plx::kBwdBN;
  if (static_cast<long long>(B) * Hq * n_qtiles > 0x7fffffffLL) return PLX_ERR_SHAPE;
  int dev = 0;
  int rc = check_arch(&dev);
  if (rc != PLX_OK) return rc;
  if ((rc = get_encoder()) != PLX_OK) return rc;
  CUtensorMap qm, rm, om, km, vm, kmq, vmq;
  const long long pq = static_cast<long long>(B) * Hq, pkv = static_cast<long long>(B) * Hkv;
  if (make_map_3d(&qm, q, d, N, pq, 16) != PLX_OK || make_map_3d(&om, dout, d, N, pq, 16) != PLX_OK ||
      make_map_3d(&km, k, d, N, pkv, plx::kBwdBN) != PLX_OK || make_map_3d(&vm, v, d, N, pkv, plx::kBwdBN) != PLX_OK ||
      make_map_3d(&kmq, k, d, N, pkv, plx::kBwdQBN) != PLX_OK || make_map_3d(&vmq, v, d, N, pkv, plx::kBwdQBN) != PLX_OK)
    return PLX_ERR_CUDA;
  if (r) {
    if (make_map_3d(&rm, r, d, N, pq, 16) != PLX_OK) return PLX_ERR_CUDA;
  } else {
    rm = qm;  // unused
  }
  const size_t half = need / 2;
  float* gbar = static_cast<float*>(workspace);
  float* dd = reinterpret_cast<float*>(static_cast<char*>(workspace) + half);
  plx::BwdParams p;
  p.dq = static_cast<__nv_bfloat16*>(dq);
  p.dr = static_cast<__nv_bfloat16*>(dr);
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.lse = lse; p.gbar = gbar; p.dd = dd; p.sbar = r ? sbar : nullptr;
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.N = N; p.G = Hq / Hkv;
  p.n_qtiles = n_qtiles; p.n_ktiles = n_ktiles;
  p.causal = causal ? 1 : 0;
  p.scale = scale;
  p.scale_log2 = scale * plx::kLog2e;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d == 128)
    return r ? launch_bwd<128, true>(qm, rm, om, km, vm, kmq, vmq, p, dout, out, obar, gbar, dd, st)
             : launch_bwd<128, false>(qm, rm, om, km, vm, kmq, vmq, p, dout, out, obar, gbar, dd, st);
  return r ? launch_bwd<64, true>(qm, rm, om, km, vm, kmq, vmq, p, dout, out, obar, gbar, dd, st)
           : launch_bwd<64, false>(qm, rm, om, km, vm, kmq, vmq, p, dout, out, obar, gbar, dd, st);
}

int plx_decode_num_splits(int B, int Hq, int Hkv, int S_max, int d) {
  if (B < 1 || Hq < 1 || Hkv < 1 || S_max < 1 || Hq % Hkv || (d != 64 && d != 128)) return decode_ctas(0, 4096);
  return plan_decode(B, Hq, Hkv, S_max, d, 0, false, false).P;
}

size_t plx_decode_workspace_size(int B, int Hq, int Hkv, int S_max, int d, int num_splits) {
  if (B < 1 || Hq < 1 || Hkv < 1 || S_max < 1 || Hq % Hkv || (d != 64 && d != 128) || num_splits < 0) return 0;
  // the paged call's plan: it covers the contiguous call too (whose segment
  // plan needs none), so one size serves both entry points
  return plan_decode(B, Hq, Hkv, S_max, d, num_splits, false, true).ws_bytes;
}

}  // extern "C"

namespace {

// plx_decode, or (rec_out) plx_decode_partial: the same validation and
// launches; rec_out receives one state record per (b, h) instead of out/lse.
int decode_common(const void* q, const void* r, const void* kcache, const void* vcache, const int32_t* seqlens,
                  void* out, float* lse, float* rec_out, int B, int Hq, int Hkv, int S_max, int d, float scale,
                  int num_splits, void* workspace, size_t workspace_bytes, void* stream, int key_offset = 0) {
  if (!q || !kcache || !vcache || !seqlens || (!out && !rec_out)) return PLX_ERR_NULL;
  if (B < 1 || Hq < 1 || Hkv < 1 || S_max < 1 || num_splits < 0) return PLX_ERR_SHAPE;
  if (d != 64 && d != 128) return PLX_ERR_HEADDIM;
  if (Hq % Hkv) return PLX_ERR_GQA;
  if (!aligned16(q) || (r && !aligned16(r)) || !aligned16(kcache) || !aligned16(vcache) ||
      (out && !aligned16(out)) || (rec_out && !aligned16(rec_out)) || (reinterpret_cast<uintptr_t>(seqlens) & 3u) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return PLX_ERR_ALIGN;
  const DecodePlan plan = plan_decode(B, Hq, Hkv, S_max, d, num_splits, rec_out != nullptr, false);
  if (plan.ws_bytes > 0 && (!workspace || workspace_bytes < plan.ws_bytes)) return PLX_ERR_WORKSPACE;
  if (plan.ws_bytes > 0 && !aligned16(workspace)) return PLX_ERR_ALIGN;
  const int G = Hq / Hkv;
  const int n_hg = (G + 7) / 8;
  if (static_cast<long long>(B) * Hkv * n_hg * ((S_max + plx::kDecTileKeys - 1) / plx::kDecTileKeys) > 0x7fffffffLL)
    return PLX_ERR_SHAPE;
  int dev = 0;
  int rc = check_arch(&dev);
  if (rc != PLX_OK) return rc;
  if ((rc = get_encoder()) != PLX_OK) return rc;

  // full 64-key tiles, and kDecTailRows-key parts for each sequence's last, partial tile
  CUtensorMap km, vm, kt, vt;
  const long long planes = static_cast<long long>(B) * Hkv;
  if (make_map_3d(&km, kcache, d, S_max, planes, plx::kDecTileKeys) != PLX_OK ||
      make_map_3d(&vm, vcache, d, S_max, planes, plx::kDecTileKeys) != PLX_OK ||
      make_map_3d(&kt, kcache, d, S_max, planes, plx::kDecTailRows) != PLX_OK ||
      make_map_3d(&vt, vcache, d, S_max, planes, plx::kDecTailRows) != PLX_OK)
    return PLX_ERR_CUDA;
  // the segment plan streams stages of its shape's height
  CUtensorMap k32, v32;
  const int seg_rows = plan.seg_many ? plx::kSegManyKeys : plx::kSegFewKeys;
  if (plan.seg && (make_map_3d(&k32, kcache, d, S_max, planes, seg_rows) != PLX_OK ||
                   make_map_3d(&v32, vcache, d, S_max, planes, seg_rows) != PLX_OK))
    return PLX_ERR_CUDA;

  plx::DecodeParams p{};
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.r = static_cast<const __nv_bfloat16*>(r);
  p.seqlens = seqlens;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = rec_out ? nullptr : lse;
  p.rec_out = rec_out;
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.S_max = S_max; p.G = G; p.n_hgroups = n_hg;
  p.rps = rows_per_slot(Hq, Hkv);
  p.ws = static_cast<float*>(workspace);
  p.chunk_tiles = plan.chunked ? plan.chunk_tiles : 0;
  p.splits = plan.chunked ? plan.splits : 0;
  p.key_offset = key_offset;
  p.scale_log2 = scale * plx::kLog2e;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d == 128)
    return r ? launch_decode<128, true, false>(km, vm, kt, vt, &k32, &v32, p, plan, st)
             : launch_decode<128, false, false>(km, vm, kt, vt, &k32, &v32, p, plan, st);
  return r ? launch_decode<64, true, false>(km, vm, kt, vt, &k32, &v32, p, plan, st)
           : launch_decode<64, false, false>(km, vm, kt, vt, &k32, &v32, p, plan, st);
}

}  // namespace

extern "C" {

int plx_decode(const void* q, const void* r, const void* kcache, const void* vcache,
               const int32_t* seqlens, void* out, float* lse, int B, int Hq, int Hkv, int S_max,
               int d, float scale, int num_splits, void* workspace, size_t workspace_bytes,
               void* stream) {
  return decode_common(q, r, kcache, vcache, seqlens, out, lse, nullptr, B, Hq, Hkv, S_max, d, scale, num_splits,
                       workspace, workspace_bytes, stream);
}

size_t plx_decode_partial_size(int B, int Hq, int Hkv, int S_max, int d, int num_splits) {
  if (B < 1 || Hq < 1 || Hkv < 1 || S_max < 1 || Hq % Hkv || (d != 64 && d != 128) || num_splits < 0) return 0;
  return align256(static_cast<size_t>(B) * Hq * (2 * d + 4) * sizeof(float)) +
         plan_decode(B, Hq, Hkv, S_max, d, num_splits, true, false).ws_bytes;
}

int plx_decode_partial(const void* q, const void* r, const void* kcache, const void* vcache,
                       const int32_t* seqlens, int key_offset, int B, int Hq, int Hkv, int S_max, int d,
                       float scale, int num_splits, float* partial, size_t partial_bytes, void* stream) {
  if (!partial) return PLX_ERR_NULL;
  if (key_offset < 0) return PLX_ERR_SHAPE;
  const size_t need = plx_decode_partial_size(B, Hq, Hkv, S_max, d, num_splits);
  if (need != 0 && partial_bytes < need) return PLX_ERR_WORKSPACE;  // bad shapes: decode_common reports them
  const size_t rec_bytes = align256(static_cast<size_t>(B > 0 ? B : 0) * (Hq > 0 ? Hq : 0) * (2 * d + 4) * sizeof(float));
  return decode_common(q, r, kcache, vcache, seqlens, nullptr, nullptr, partial, B, Hq, Hkv, S_max, d, scale,
                       num_splits, reinterpret_cast<char*>(partial) + rec_bytes,
                       partial_bytes > rec_bytes ? partial_bytes - rec_bytes : 0, stream, key_offset);
}

// out / lse of `rows` rows from `blocks` blocks of state records, each block
// [rows, 2d + 4] (the merge over context-parallel ranks or key chunks)
static int merge_common(const float* recs, int blocks, long long rows, int d, void* out, float* lse, void* stream) {
  if (!recs || !out) return PLX_ERR_NULL;
  if (blocks < 1 || rows < 1) return PLX_ERR_SHAPE;
  if (d != 64 && d != 128) return PLX_ERR_HEADDIM;
  if (!aligned16(recs) || (reinterpret_cast<uintptr_t>(out) & 7u) || (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return PLX_ERR_ALIGN;
  const long long threads = rows * (d / 4);
  if ((threads + 255) / 256 > 0x7fffffffLL) return PLX_ERR_SHAPE;
  int dev = 0;
  int rc = check_arch(&dev);
  if (rc != PLX_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const unsigned grid = static_cast<unsigned>((threads + 255) / 256);
  const long long rf = 2 * d + 4;
  if (d == 128)
    plx::plx_record_merge_kernel<128><<<grid, 256, 0, st>>>(recs, blocks, rows, static_cast<__nv_bfloat16*>(out), lse,
                                                           rows * rf, rf);
  else
    plx::plx_record_merge_kernel<64><<<grid, 256, 0, st>>>(recs, blocks, rows, static_cast<__nv_bfloat16*>(out), lse,
                                                          rows * rf, rf);
  return cudaGetLastError() == cudaSuccess ? PLX_OK : PLX_ERR_CUDA;
}

int plx_decode_merge(const float* partials, int ranks, int B, int Hq, int d, void* out, float* lse, void* stream) {
  if (B < 1 || Hq < 1) return (!partials || !out) ? PLX_ERR_NULL : PLX_ERR_SHAPE;
  return merge_common(partials, ranks, static_cast<long long>(B) * Hq, d, out, lse, stream);
}

int plx_fwd_merge(const float* partials, int ranks, int B, int Hq, int N, int d, void* out, float* lse,
                  void* stream) {
  if (B < 1 || Hq < 1 || N < 1) return (!partials || !out) ? PLX_ERR_NULL : PLX_ERR_SHAPE;
  return merge_common(partials, ranks, static_cast<long long>(B) * Hq * N, d, out, lse, stream);
}

int plx_check_device_status(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return PLX_ERR_CUDA;
  unsigned int word = 0;
  if (cudaMemcpyFromSymbol(&word, g_plx_error, sizeof(word)) != cudaSuccess) return PLX_ERR_CUDA;
  if (word == 0u) return PLX_OK;
  const unsigned int zero = 0u;
  if (cudaMemcpyToSymbol(g_plx_error, &zero, sizeof(zero)) != cudaSuccess) return PLX_ERR_CUDA;
  return PLX_ERR_DEVICE_TIMEOUT;
}

}  // extern "C"

namespace {
// One mbarrier that expects one arrival which never comes: the wait runs out.
__global__ void plx_selftest_wait_kernel(long long limit) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    plx::mbar_init(plx::smem_u32(&bar), 1);
    plx::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool ok = plx::mbar_wait(plx::smem_u32(&bar), 0, plx::kErrSelftest, limit);
    if (ok) plx::set_error(0xDEADu);  // cannot happen: nothing arrives
  }
}
}  // namespace

extern "C" int plx_selftest_wait_timeout(unsigned long long limit_cycles, void* stream) {
  int dev = 0;
  int rc = check_arch(&dev);
  if (rc != PLX_OK) return rc;
  if (limit_cycles > (1ULL << 32)) return PLX_ERR_SHAPE;  // keep the test short (~2 s max)
  plx_selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<long long>(limit_cycles));
  return cudaGetLastError() == cudaSuccess ? PLX_OK : PLX_ERR_CUDA;
}

// ------------------------------------------------------------------ no-alloc decode
// Scratch for plx_decode_noalloc: a fixed device array, zero-initialised at
// module load and shared by every call.  In host code the symbol is only a
// stand-in; its device address is looked up once per device.
static __device__ __align__(256) unsigned char g_plx_noalloc_scratch[PLX_NOALLOC_SCRATCH_BYTES];

namespace {
void* g_noalloc_ptr[kMaxDevices];
std::mutex g_noalloc_mu;
}  // namespace

extern "C" int plx_decode_noalloc(const void* q, const void* r, const void* kcache, const void* vcache,
                                  const int32_t* seqlens, void* out, float* lse, int B, int Hq, int Hkv,
                                  int S_max, int d, float scale, int num_splits, void* stream) {
  if (B < 1 || Hq < 1 || Hkv < 1 || S_max < 1 || num_splits < 0) return PLX_ERR_SHAPE;
  if (d != 64 && d != 128) return PLX_ERR_HEADDIM;
  if (Hq % Hkv) return PLX_ERR_GQA;
  const size_t need = plx_decode_workspace_size(B, Hq, Hkv, S_max, d, num_splits);
  if (need > PLX_NOALLOC_SCRATCH_BYTES) return PLX_ERR_WORKSPACE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PLX_ERR_CUDA;
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
      void* ptr = nullptr;
      if (cudaGetSymbolAddress(&ptr, g_plx_noalloc_scratch) != cudaSuccess || ptr == nullptr)
        return PLX_ERR_CUDA;
      g_noalloc_ptr[dev] = ptr;
    }
    scratch = g_noalloc_ptr[dev];
  }
  return plx_decode(q, r, kcache, vcache, seqlens, out, lse, B, Hq, Hkv, S_max, d, scale, num_splits,
                    scratch, PLX_NOALLOC_SCRATCH_BYTES, stream);
}

// ------------------------------------------------------------------ q, k, v, rho projection
namespace {

int proj_common(const void* x, const void* w, plx::ProjParams& p, int M, int d_model, void* stream) {
  if (!x || !w) return PLX_ERR_NULL;
  if (M < 1 || d_model < 8 || d_model % 8 || p.Hq < 1 || p.Hkv < 1) return PLX_ERR_SHAPE;
  if (p.d != 64 && p.d != 128) return PLX_ERR_HEADDIM;
  if (p.Hq % p.Hkv) return PLX_ERR_GQA;
  if (!aligned16(x) || !aligned16(w)) return PLX_ERR_ALIGN;
  const long long nout = static_cast<long long>(2 * p.Hkv + (p.r ? 2 : 1) * p.Hq) * p.d;
  const long long m_tiles = (M + plx::kPjBM - 1) / plx::kPjBM;
  long long n_tiles = (nout + 63) / 64;
  if (m_tiles * n_tiles > 0x7fffffffLL || static_cast<long long>(M) * nout > (1LL << 40)) return PLX_ERR_SHAPE;
  int dev = 0;
  int rc = check_arch(&dev);
  if (rc != PLX_OK) return rc;
  if ((rc = get_encoder()) != PLX_OK) return rc;
  // few rows (a decode step): narrow tiles, so that more CTAs share the weight stream
  const bool narrow = M <= plx::kPjBM;
  const int bn = narrow ? 64 : 256;
  n_tiles = (nout + bn - 1) / bn;
  CUtensorMap xm, wm;
  if (make_map_2d(&xm, x, d_model, M, plx::kPjBM) != PLX_OK || make_map_2d(&wm, w, d_model, nout, bn) != PLX_OK)
    return PLX_ERR_CUDA;
  p.M = M;
  p.K = d_model;
  p.Nout = static_cast<int>(nout);
  p.m_tiles = static_cast<int>(m_tiles);
  p.n_tiles = static_cast<int>(n_tiles);
  p.num_tiles = static_cast<int>(m_tiles * n_tiles);
  p.k_steps = (d_model + plx::kPjBK - 1) / plx::kPjBK;
  const unsigned grid = static_cast<unsigned>(std::min<long long>(p.num_tiles, g_sm_count[dev]));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (narrow) {
    static bool done[kMaxDevices];
    auto kern = plx::plx_proj_kernel<64>;
    if (ensure_smem(kern, plx::ProjCfg<64>::kSmemBytes, &done[dev]) != PLX_OK) return PLX_ERR_CUDA;
    kern<<<grid, plx::kPjThreads, plx::ProjCfg<64>::kSmemBytes, st>>>(xm, wm, p);
  } else {
    static bool done[kMaxDevices];
    auto kern = plx::plx_proj_kernel<256>;
    if (ensure_smem(kern, plx::ProjCfg<256>::kSmemBytes, &done[dev]) != PLX_OK) return PLX_ERR_CUDA;
    kern<<<grid, plx::kPjThreads, plx::ProjCfg<256>::kSmemBytes, st>>>(xm, wm, p);
  }
  return cudaGetLastError() == cudaSuccess ? PLX_OK : PLX_ERR_CUDA;
}

}  // namespace

extern "C" {

int plx_qkvr_proj(const void* x, const void* w, void* q, void* k, void* v, void* r, int B, int N, int d_model,
                  int Hq, int Hkv, int d, void* stream) {
  if (!q || !k || !v) return PLX_ERR_NULL;
  if (B < 1 || N < 1) return PLX_ERR_SHAPE;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || (r && !aligned16(r))) return PLX_ERR_ALIGN;
  if (static_cast<long long>(B) * N > 0x7fffffffLL) return PLX_ERR_SHAPE;
  plx::ProjParams p{};
  p.q = static_cast<__nv_bfloat16*>(q);
  p.k = static_cast<__nv_bfloat16*>(k);
  p.v = static_cast<__nv_bfloat16*>(v);
  p.r = static_cast<__nv_bfloat16*>(r);
  p.N = N; p.Hq = Hq; p.Hkv = Hkv; p.d = d;
  return proj_common(x, w, p, B * N, d_model, stream);
}

int plx_qkvr_proj_decode(const void* x, const void* w, void* q, void* r, void* kcache, void* vcache,
                         const int32_t* seqlens, int32_t* seqlens_out, int B, int d_model, int Hq, int Hkv,
                         int S_max, int d, void* stream) {
  if (!q || !kcache || !vcache || !seqlens) return PLX_ERR_NULL;
  if (B < 1 || S_max < 1) return PLX_ERR_SHAPE;
  if (seqlens_out && static_cast<const void*>(seqlens_out) == static_cast<const void*>(seqlens)) return PLX_ERR_SHAPE;
  if (!aligned16(q) || (r && !aligned16(r)) || !aligned16(kcache) || !aligned16(vcache) ||
      (reinterpret_cast<uintptr_t>(seqlens) & 3u) || (reinterpret_cast<uintptr_t>(seqlens_out) & 3u))
    return PLX_ERR_ALIGN;
  plx::ProjParams p{};
  p.q = static_cast<__nv_bfloat16*>(q);
  p.r = static_cast<__nv_bfloat16*>(r);
  p.decode = 1;
  p.kcache = static_cast<__nv_bfloat16*>(kcache);
  p.vcache = static_cast<__nv_bfloat16*>(vcache);
  p.S_max = S_max;
  p.seqlens = seqlens;
  p.seqlens_out = seqlens_out;
  p.N = 1; p.Hq = Hq; p.Hkv = Hkv; p.d = d;
  return proj_common(x, w, p, B, d_model, stream);
}

int plx_qkvr_proj_decode_paged(const void* x, const void* w, void* q, void* r, void* kpool, void* vpool,
                               const int32_t* block_table, const int32_t* seqlens, int32_t* seqlens_out, int B,
                               int d_model, int Hq, int Hkv, int num_pages, int page_size, int max_pages, int d,
                               void* stream) {
  if (!q || !kpool || !vpool || !seqlens || !block_table) return PLX_ERR_NULL;
  if (B < 1 || num_pages < 1 || max_pages < 1) return PLX_ERR_SHAPE;
  if (page_size < 16 || page_size > 4096 || (page_size & (page_size - 1))) return PLX_ERR_SHAPE;
  if (static_cast<long long>(max_pages) * page_size > 0x7fffffffLL) return PLX_ERR_SHAPE;
  if (seqlens_out && static_cast<const void*>(seqlens_out) == static_cast<const void*>(seqlens)) return PLX_ERR_SHAPE;
  if (!aligned16(q) || (r && !aligned16(r)) || !aligned16(kpool) || !aligned16(vpool) ||
      (reinterpret_cast<uintptr_t>(seqlens) & 3u) || (reinterpret_cast<uintptr_t>(seqlens_out) & 3u) ||
      (reinterpret_cast<uintptr_t>(block_table) & 3u))
    return PLX_ERR_ALIGN;
  plx::ProjParams p{};
  p.q = static_cast<__nv_bfloat16*>(q);
  p.r = static_cast<__nv_bfloat16*>(r);
  p.decode = 1;
  p.kcache = static_cast<__nv_bfloat16*>(kpool);
  p.vcache = static_cast<__nv_bfloat16*>(vpool);
  p.seqlens = seqlens;
  p.seqlens_out = seqlens_out;
  p.block_table = block_table;
  p.num_pages = num_pages;
  p.page_size = page_size;
  int shift = 0;
  while ((1 << shift) < page_size) ++shift;
  p.page_shift = shift;
  p.max_pages = max_pages;
  p.N = 1; p.Hq = Hq; p.Hkv = Hkv; p.d = d;
  return proj_common(x, w, p, B, d_model, stream);
}

}  // extern "C"
