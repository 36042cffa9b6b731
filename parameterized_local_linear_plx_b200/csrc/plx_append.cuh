// plx_append.cuh -- decode-time KV append: the new token's key and value of
// every KV head go into the cache at position seqlens[b] (the slot after the
// live keys), before the decode step that attends them.  The pages describe
// a KV cache that grows by one token per step (zubnet.ai, Parallax page: the
// method keeps a KV cache like softmax attention); this is that step.
//
// One warp per batch entry: it reads the entry's length once, copies the
// d-element k and v rows of every KV head with 16-byte stores, and then (if
// asked) advances the length -- no other warp touches that entry.  An entry
// whose slot is past the cache (seqlens[b] >= capacity, a negative length, or
// a page id outside the pool) is not written, and its length is not advanced.
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

namespace plx {

struct AppendParams {
  const __nv_bfloat16* knew;   // [B, Hkv, D]
  const __nv_bfloat16* vnew;   // [B, Hkv, D]
  __nv_bfloat16* kcache;       // contiguous [B, Hkv, S_max, D] or pool [num_pages, Hkv, page_size, D]
  __nv_bfloat16* vcache;
  int32_t* seqlens;            // [B] (read; advanced by one when advance != 0)
  const int32_t* block_table;  // [B, max_pages] or nullptr (contiguous)
  int B, Hkv, S_max, num_pages, page_size, page_shift, max_pages, advance;
};

template <int D>
__global__ void __launch_bounds__(256) plx_kv_append_kernel(const AppendParams p) {
  const int b = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (b >= p.B) return;
  const int pos = p.seqlens[b];
  bool ok = pos >= 0;
  size_t base = 0;  // element offset of (b or page, head 0, slot) in the cache
  size_t head_stride = 0;
  if (p.block_table == nullptr) {
    ok = ok && pos < p.S_max;
    base = (static_cast<size_t>(b) * p.Hkv * p.S_max + pos) * D;
    head_stride = static_cast<size_t>(p.S_max) * D;
  } else {
    ok = ok && pos < p.max_pages * p.page_size;
    if (ok) {
      const int pg = p.block_table[static_cast<size_t>(b) * p.max_pages + (pos >> p.page_shift)];
      ok = pg >= 0 && pg < p.num_pages;
      base = (static_cast<size_t>(pg) * p.Hkv * p.page_size + (pos & (p.page_size - 1))) * D;
      head_stride = static_cast<size_t>(p.page_size) * D;
    }
  }
  if (ok) {
    constexpr int kVec = D / 8;  // 16-byte vectors per row
    for (int i = lane; i < p.Hkv * kVec; i += 32) {
      const int g = i / kVec, c = i % kVec;
      const size_t src = (static_cast<size_t>(b) * p.Hkv + g) * D;
      const size_t dst = base + g * head_stride;
      reinterpret_cast<uint4*>(p.kcache + dst)[c] = reinterpret_cast<const uint4*>(p.knew + src)[c];
      reinterpret_cast<uint4*>(p.vcache + dst)[c] = reinterpret_cast<const uint4*>(p.vnew + src)[c];
    }
  }
  __syncwarp();  // every lane has read the length before it changes
  if (p.advance && lane == 0 && ok) p.seqlens[b] = pos + 1;
}

}  // namespace plx
