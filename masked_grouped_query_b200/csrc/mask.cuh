// mask.cuh -- the visibility rule and the key-range arithmetic shared by the
// host planner and the kernels of this library (not by the oracle).
//
// Query row i of a q_len-row block sits at position qpos = kv_len - q_len + i
// (bottom-right alignment).  Key j is visible iff
//   j < kv_len && (!causal || j <= qpos) && (window <= 0 || 0 <= qpos - j < window).
// For one qpos the visible keys therefore form the interval
//   [first_key(qpos), last_key(qpos)], empty when last < first,
// and both ends are non-decreasing in qpos.
#pragma once

#include <stdint.h>

namespace gqa {

struct MaskSpec {
  int q_len;
  int kv_len;
  int causal;
  int window;  // <= 0: none
};

__host__ __device__ __forceinline__ int first_key(const MaskSpec& m, int qpos) {
  if (m.window > 0) {
    long long f = (long long)qpos - m.window + 1;
    return f > 0 ? (int)f : 0;
  }
  return 0;
}

__host__ __device__ __forceinline__ int last_key(const MaskSpec& m, int qpos) {
  if (m.causal || m.window > 0) return qpos < m.kv_len - 1 ? qpos : m.kv_len - 1;
  return m.kv_len - 1;
}

// Smallest and largest query position among rows [r0, r0 + n) of a row block
// in which row r is query i = r % q_len (rows of consecutive q heads follow
// each other).
__host__ __device__ __forceinline__ void qpos_span(const MaskSpec& m, long long r0, int n,
                                                   int& qmin, int& qmax) {
  const int base = m.kv_len - m.q_len;
  if (n >= m.q_len) {
    qmin = base;
    qmax = base + m.q_len - 1;
    return;
  }
  const int i0 = (int)(r0 % m.q_len);
  const int i1 = (int)((r0 + n - 1) % m.q_len);
  if (i1 >= i0) {
    qmin = base + i0;
    qmax = base + i1;
  } else {  // wraps into the next head: every position occurs
    qmin = base;
    qmax = base + m.q_len - 1;
  }
}

// Key tiles of `tile` keys that rows [r0, r0+n) may touch:
// tiles [t_first, t_first + t_count).  t_count == 0 when no key is visible.
// Also returns the key interval every one of these rows sees
// (all_lo..all_hi, empty when all_hi < all_lo): tiles inside it need no mask.
struct KeyRange {
  int t_first, t_count;
  int all_lo, all_hi;
  int any_lo, any_hi;
};

// Tiles here start at key k_base (tile t holds keys k_base + tile*t ..);
// k_base <= every visible key.  key_range is the k_base = 0 case.
__host__ __device__ __forceinline__ KeyRange key_range_from(const MaskSpec& m, long long r0, int n,
                                                            int tile, int k_base) {
  KeyRange kr;
  int qmin, qmax;
  qpos_span(m, r0, n, qmin, qmax);
  kr.any_lo = first_key(m, qmin);
  kr.any_hi = last_key(m, qmax);
  kr.all_lo = first_key(m, qmax);
  kr.all_hi = last_key(m, qmin);
  if (m.kv_len <= 0 || kr.any_hi < kr.any_lo) {
    kr.t_first = 0;
    kr.t_count = 0;
  } else {
    kr.t_first = (kr.any_lo - k_base) / tile;
    kr.t_count = (kr.any_hi - k_base) / tile - kr.t_first + 1;
  }
  return kr;
}

__host__ __device__ __forceinline__ KeyRange key_range(const MaskSpec& m, long long r0, int n,
                                                       int tile) {
  return key_range_from(m, r0, n, tile, 0);
}

// Ring (circular) K/V storage: key j of a kv_len-key sequence lives in slot
// j % slots of a ring of `slots` slots (a multiple of `tile`), so the ring
// holds keys [kv_len - slots, kv_len) once it has wrapped.  Cut the keys
// into tiles aligned to the ring's slot tiles: with w = kv_len % slots,
// tile t holds keys k_base + tile*t .. + tile - 1 where
// k_base = kv_len - slots - (w % tile), and sits in ring slot tile
// (w / tile + t) % (slots / tile).  Only the first and last of these tiles
// share a slot tile; each also covers keys that are not in the ring (older
// than kv_len - slots, or past kv_len), which callers must keep hidden.
__host__ __device__ __forceinline__ int ring_k_base(int kv_len, int slots, int tile) {
  const int w = kv_len % slots;
  return kv_len - slots - (w % tile);
}
__host__ __device__ __forceinline__ int ring_phase(int kv_len, int slots, int tile) {
  return (kv_len % slots) / tile;
}

}  // namespace gqa
