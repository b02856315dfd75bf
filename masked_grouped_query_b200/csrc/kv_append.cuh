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

// ------------------------------------------------------------ staged runs
// When the cache and the new tokens share their layout ([B][S][H][D] cache
// with [B][L][H][D] tokens, or [B][H][S][D] with [B][H][L][D]) and a ring
// does not wrap inside the block, the L new tokens of one batch row (one
// (batch, head) row in the head-major case) are one contiguous run of
// elements in the source AND in the cache.  Those runs are cut into chunks of
// kRunChunk elements; each persistent CTA takes every gridDim.x-th chunk
// (keys first, then values).  Thread 0 streams source chunks into a ring of
// kRunStages shared-memory stages with one bulk copy per chunk (no per-thread
// load instructions, many bytes in flight per SM); all threads convert a
// chunk from shared memory and write it to the cache with coalesced 16-byte
// stores.  Bytes moved are the same as in the generic kernel.
struct KvRunParams {
  void* k_cache;
  void* v_cache;
  const void* new_k;
  const void* new_v;
  uint32_t runs;            // runs per tensor
  uint32_t run_len;         // elements per run (a multiple of 8)
  uint32_t chunks_per_run;  // ceil(run_len / kRunChunk)
  uint64_t src_run_stride;  // elements between run starts in the source
  uint64_t dst_run_stride;  // elements between run starts in the cache
  uint64_t dst_first;       // cache element offset of run 0's first element
};

constexpr int kRunChunk = 4096;  // elements per chunk: 16 KB of fp32, 8 KB of bf16
constexpr int kRunStages = 4;
constexpr int kRunCtasPerSm = 2;
constexpr int kRunThreads = 256;  // each thread converts two groups of 8 elements

template <bool kNewF32>
constexpr uint32_t run_stage_bytes() {
  return kRunChunk * (kNewF32 ? 4u : 2u);
}
template <bool kNewF32>
constexpr uint32_t run_smem_bytes() {
  return kRunStages * run_stage_bytes<kNewF32>() + kRunStages * 8u;
}

// Chunk `item` of the flat (tensor, run, chunk) order: source and cache
// addresses of its first element and its length in elements.
template <bool kNewF32, bool kCacheF32>
__device__ __forceinline__ void kv_run_locate(const KvRunParams& p, uint32_t item,
                                              uint32_t per_tensor, const char*& src, char*& dst,
                                              uint32_t& len) {
  const bool values = item >= per_tensor;
  const uint32_t e = values ? item - per_tensor : item;
  const uint32_t run = e / p.chunks_per_run, c = e % p.chunks_per_run;
  const uint32_t off = c * (uint32_t)kRunChunk;
  len = min((uint32_t)kRunChunk, p.run_len - off);
  src = static_cast<const char*>(values ? p.new_v : p.new_k) +
        ((uint64_t)run * p.src_run_stride + off) * (kNewF32 ? 4 : 2);
  dst = static_cast<char*>(values ? p.v_cache : p.k_cache) +
        ((uint64_t)run * p.dst_run_stride + p.dst_first + off) * (kCacheF32 ? 4 : 2);
}

// Converts group g (8 elements) of a staged chunk and stores it.
template <bool kNewF32, bool kCacheF32>
__device__ __forceinline__ void kv_run_group(const uint8_t* stage, char* dst, uint32_t g) {
  if constexpr (kNewF32) {
    const uint4 a = reinterpret_cast<const uint4*>(stage)[2 * g];
    const uint4 b = reinterpret_cast<const uint4*>(stage)[2 * g + 1];
    if constexpr (kCacheF32) {
      reinterpret_cast<uint4*>(dst)[2 * g] = a;
      reinterpret_cast<uint4*>(dst)[2 * g + 1] = b;
    } else {
      reinterpret_cast<uint4*>(dst)[g] = make_uint4(
          pack_bf16(__uint_as_float(a.x), __uint_as_float(a.y)),
          pack_bf16(__uint_as_float(a.z), __uint_as_float(a.w)),
          pack_bf16(__uint_as_float(b.x), __uint_as_float(b.y)),
          pack_bf16(__uint_as_float(b.z), __uint_as_float(b.w)));
    }
  } else {
    const uint4 a = reinterpret_cast<const uint4*>(stage)[g];
    if constexpr (kCacheF32) {
      reinterpret_cast<uint4*>(dst)[2 * g] =
          make_uint4(a.x << 16, a.x & 0xffff0000u, a.y << 16, a.y & 0xffff0000u);
      reinterpret_cast<uint4*>(dst)[2 * g + 1] =
          make_uint4(a.z << 16, a.z & 0xffff0000u, a.w << 16, a.w & 0xffff0000u);
    } else {
      reinterpret_cast<uint4*>(dst)[g] = a;
    }
  }
}

// Two CTAs per SM (measured: 4 stages x 2 CTAs beat 8 or 12 stages x 1 CTA
// and 8 KB chunks).  Every thread takes the same loop trips; a bounded wait
// that gives up is seen by all threads through __syncthreads_or, so the CTA
// leaves together (no thread is left at a barrier).
template <bool kNewF32, bool kCacheF32>
__global__ void __launch_bounds__(kRunThreads, kRunCtasPerSm) kv_append_runs_kernel(const KvRunParams p) {
  constexpr uint32_t kStage = run_stage_bytes<kNewF32>();
  extern __shared__ __align__(128) uint8_t run_smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(run_smem + kRunStages * kStage);
  const uint32_t per_tensor = p.runs * p.chunks_per_run;
  const uint32_t items = 2 * per_tensor;

  auto issue = [&](uint32_t j) {  // thread 0: stage the CTA's j-th chunk
    const uint32_t item = blockIdx.x + j * gridDim.x;
    if (item >= items) return;
    const char* src;
    char* dst;
    uint32_t len;
    kv_run_locate<kNewF32, kCacheF32>(p, item, per_tensor, src, dst, len);
    const uint32_t bytes = len * (kNewF32 ? 4u : 2u);
    uint64_t* bar = &full[j % kRunStages];
    mbar_arrive_expect_tx(bar, bytes);
    bulk_load(run_smem + (j % kRunStages) * kStage, src, bytes, bar);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRunStages; ++s) mbar_init(&full[s], 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0)
    for (uint32_t j = 0; j < (uint32_t)kRunStages; ++j) issue(j);

  for (uint32_t j = 0; blockIdx.x + j * gridDim.x < items; ++j) {
    const uint32_t item = blockIdx.x + j * gridDim.x;
    const int s = j % kRunStages;
    const bool ok = mbar_wait(&full[s], (j / kRunStages) & 1u, kStatusTimeoutConsumer);
    if (ok) {
      const char* src;
      char* dst;
      uint32_t len;
      kv_run_locate<kNewF32, kCacheF32>(p, item, per_tensor, src, dst, len);
      const uint8_t* stage = run_smem + s * kStage;
      const uint32_t groups = len / 8;
#pragma unroll
      for (uint32_t h = 0; h < 2; ++h) {
        const uint32_t g = threadIdx.x + h * kRunThreads;
        if (g < groups) kv_run_group<kNewF32, kCacheF32>(stage, dst, g);
      }
    }
    // every thread is done with stage s before it is refilled
    if (__syncthreads_or(!ok)) break;
    if (threadIdx.x == 0) issue(j + kRunStages);
  }
}

}  // namespace gqa
