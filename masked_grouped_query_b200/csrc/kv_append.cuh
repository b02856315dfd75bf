// kv_append.cuh -- write the keys and values of L new tokens into a key cache
// and a value cache at slots [position, position + L) ("KV Cache Update at a
// Position", TensorTonic: in every batch row and head the new vectors land in
// order at those slots, converted to the cache dtype; every other slot keeps
// its contents).
//
// Caches: bf16 or fp32, laid out [batch][slots][heads][D] (the page's layout)
// or [batch][heads][slots][D] (the attention kernels' native layout).  New
// tokens: fp32 (the page's) or bf16, [batch][L][heads][D] or
// [batch][heads][L][D].  fp32 -> bf16 rounds to nearest even.
//
// One thread moves 8 consecutive elements of one (batch, token, head) row,
// so every 16- or 32-byte access is aligned and a warp covers whole rows:
// the kernel is a strided copy, bound by HBM bandwidth (bytes read + bytes
// written), with a grid-stride loop over one wave of resident blocks and
// 32-bit index arithmetic.
#pragma once

#include "ptx.cuh"

namespace gqa {

struct KvAppendParams {
  void* k_cache;
  void* v_cache;
  const void* new_k;
  const void* new_v;
  int batch, heads, slots, head_dim, position, count;  // count = L
  int cache_seq_major;  // 1: [B][S][H][D], 0: [B][H][S][D]
  int ring;             // 1: token position + l goes to slot (position + l) % slots
  int new_head_major;   // 1: [B][H][L][D], 0: [B][L][H][D]
};

// Moves chunk i (8 elements; keys for i < n, values after) of the new tokens.
template <bool kNewF32, bool kCacheF32>
__device__ __forceinline__ void kv_append_locate(const KvAppendParams& p, uint32_t i, uint32_t n,
                                                 uint32_t d8, const void*& src, void*& dst) {
  const bool values = i >= n;
  const uint32_t e = values ? i - n : i;
  const uint32_t c = e % d8, src_row = e / d8;
  // src_row enumerates the new tokens' rows in their own order
  const uint32_t inner = p.new_head_major ? p.count : p.heads;
  const uint32_t a = src_row % inner, rest = src_row / inner;
  const uint32_t outer = p.new_head_major ? p.heads : p.count;
  const uint32_t bb = rest / outer, o = rest % outer;
  const uint32_t l = p.new_head_major ? a : o, h = p.new_head_major ? o : a;
  const uint32_t slot = p.ring ? (uint32_t)(((long long)p.position + l) % p.slots)
                              : (uint32_t)p.position + l;
  const uint64_t dst_row = p.cache_seq_major
                               ? ((uint64_t)bb * p.slots + slot) * p.heads + h
                               : ((uint64_t)bb * p.heads + h) * p.slots + slot;
  const uint64_t src_off = (uint64_t)src_row * p.head_dim + 8 * c;
  const uint64_t dst_off = dst_row * p.head_dim + 8 * c;
  src = static_cast<const char*>(values ? p.new_v : p.new_k) + src_off * (kNewF32 ? 4 : 2);
  dst = static_cast<char*>(values ? p.v_cache : p.k_cache) + dst_off * (kCacheF32 ? 4 : 2);
}

// Every chunk index fits in 32 bits (the host rejects larger blocks).  Each
// thread takes kUnroll chunks a grid-stride apart and issues all their loads
// before any store, so several 16/32-byte loads are in flight per thread.
template <bool kNewF32, bool kCacheF32>
__global__ void __launch_bounds__(256) kv_append_kernel(const KvAppendParams p) {
  constexpr int kUnroll = 4;
  const uint32_t d8 = (uint32_t)p.head_dim / 8;
  const uint32_t n = (uint32_t)p.batch * p.heads * p.count * d8;
  const uint32_t total = 2 * n;
  const uint32_t stride = gridDim.x * blockDim.x;
  for (uint32_t i0 = blockIdx.x * blockDim.x + threadIdx.x; i0 < total;
       i0 += kUnroll * stride) {
    uint4 w[kUnroll][kNewF32 ? 2 : 1];
    void* dst[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const uint32_t i = i0 + u * stride;
      dst[u] = nullptr;
      if (i < total) {
        const void* src;
        kv_append_locate<kNewF32, kCacheF32>(p, i, n, d8, src, dst[u]);
        w[u][0] = __ldcs(reinterpret_cast<const uint4*>(src));  // read once: streaming
        if constexpr (kNewF32) w[u][1] = __ldcs(reinterpret_cast<const uint4*>(src) + 1);
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      if (!dst[u]) continue;
      if constexpr (kNewF32 && !kCacheF32) {
        const uint4 a = w[u][0], b = w[u][1];
        *reinterpret_cast<uint4*>(dst[u]) = make_uint4(
            pack_bf16(__uint_as_float(a.x), __uint_as_float(a.y)),
            pack_bf16(__uint_as_float(a.z), __uint_as_float(a.w)),
            pack_bf16(__uint_as_float(b.x), __uint_as_float(b.y)),
            pack_bf16(__uint_as_float(b.z), __uint_as_float(b.w)));
      } else if constexpr (kNewF32 && kCacheF32) {
        reinterpret_cast<uint4*>(dst[u])[0] = w[u][0];
        reinterpret_cast<uint4*>(dst[u])[1] = w[u][1];
      } else if constexpr (!kNewF32 && kCacheF32) {
        // bf16 -> fp32 is exact: the bf16 bits become the top half.
        const uint4 a = w[u][0];
        reinterpret_cast<uint4*>(dst[u])[0] =
            make_uint4(a.x << 16, a.x & 0xffff0000u, a.y << 16, a.y & 0xffff0000u);
        reinterpret_cast<uint4*>(dst[u])[1] =
            make_uint4(a.z << 16, a.z & 0xffff0000u, a.w << 16, a.w & 0xffff0000u);
      } else {
        *reinterpret_cast<uint4*>(dst[u]) = w[u][0];
      }
    }
  }
}

}  // namespace gqa
