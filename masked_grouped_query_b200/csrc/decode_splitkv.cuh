// decode_splitkv.cuh -- memory-bound split-KV attention for short query
// blocks (decode and multi-token decode), sm_100a.
//
// Work unit: one kv head of one batch element (b, kvh) and a block of up to
// 64 "rows" -- the q rows of every q head of that GQA group, packed so each
// K/V tile feeds all of them (the decode shapes with GQA ratios 1:1 to 16:1
// of "TPU v6e Masked GQA Kernel Optimization", "What You Have").  The key
// range of a row block is cut into `splits` chunks; one CTA per chunk.
//
// Per CTA: one loader warp streams 64-key K and V tiles with TMA
// (cp.async.bulk.tensor, 128-byte swizzle) into a ring of 3 stages (2 for
// head_dim above 128; 5 when the grid has at most one CTA per SM, see
// DecodeCfg) guarded by mbarriers;
// four compute warps run S = Q K^T and O += P V on the tensor cores with
// mma.sync m16n8k16 (bf16 in, fp32 accumulate) and an online fp32 softmax
// with the softcap and mask fused in.  Chunks end with a log-sum-exp partial
// (o_s, lse_s); the last CTA of a row block to finish (a ticket counter, no
// waiting) merges the partials in fixed split order -- deterministic -- and
// writes bf16 o.  A row with no visible key comes out as zeros.
#pragma once

#include "mask.cuh"
#include "ptx.cuh"

namespace gqa {

constexpr int kDecTile = 64;        // keys per pipeline stage
constexpr int kDecRows = 64;        // rows per CTA (at most)
constexpr int kDecComputeWarps = 4;
constexpr int kDecThreads = 32 * (kDecComputeWarps + 1);

struct DecodeParams {
  const __nv_bfloat16* q;
  __nv_bfloat16* o;
  int q_len, kv_len, head_dim;
  int kv_heads;        // K/V maps are 4-D: (col, key, kv head, batch)
  int k_base;          // key of tile 0's first column (0, or the ring's key base)
  int ring_tiles;      // ring: slots / 64 (tile t is in slot tile (ring_phase + t) % ring_tiles); 0: none
  int ring_phase;
  // Fused KV-cache append (app_count > 0): before loading its key tiles, a
  // CTA writes the new tokens that fall in them into the caches (token l is
  // key app_pos + l, slot (app_pos + l) % app_slots for a ring).
  int app_count, app_pos, app_slots, app_ring;
  int app_new_f32, app_new_head_major, app_cache_seq_major;
  const void* app_new_k;
  const void* app_new_v;
  __nv_bfloat16* app_k_cache;
  __nv_bfloat16* app_v_cache;
  int rows;            // rows per (b, kvh): group * q_len
  int row_blocks;      // ceil(rows / 64)
  int block_rows;      // min(64, rows): row stride of the partial buffers
  int causal, window;
  int use_softcap;
  float logit_scale;   // log2(e) / sqrt(D)            (no softcap)
  float cap_in;        // 1 / (sqrt(D) * softcap)       (softcap)
  float cap_out;       // softcap * log2(e)             (softcap)
  int splits;          // chunks per (unit, row block)
  int tiles_per_split;
  float* part_o;       // [unit][rb][split][block_rows][head_dim]  (o_s, normalised)
  float* part_lse;     // [unit][rb][split][block_rows]            (log2 domain)
  unsigned int* tickets;  // [unit][rb], zero between calls
};

// kDeep: a 5-stage ring (160 KB in flight for KS = 8) for grids of at most
// one CTA per SM, where the 3-stage ring of two co-resident CTAs would leave
// each SM with half the bytes in flight.
template <int KS, bool kDeep = false>
struct DecodeCfg {
  static constexpr int kDChunks = KS / 4;                 // 64-column TMA boxes
  static constexpr int kBoxBytes = kDecTile * 128;        // one 64-key x 64-col box
  static constexpr int kTileBytes = kDChunks * kBoxBytes; // K (or V) tile
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kStages = kDeep ? 5 : KS <= 8 ? 3 : 2;
  static constexpr int kRingBytes = kStages * kStageBytes;
  static constexpr int kMergeBytes = kDecComputeWarps * 16 * (KS * 16 + 2) * 4;
  static constexpr int kSmemBytes =
      1024 + (kRingBytes > kMergeBytes ? kRingBytes : kMergeBytes) + 2 * kStages * 8 + 64;
};

// kT = true: the variant for row blocks of at most 8 rows (single-token GQA
// decode).  Keys become the M dimension of the tensor-core tiles --
// S^T = K Q^T (m16 keys x n8 rows) and O^T += V^T P^T (m16 head-dim x n8
// rows), with P^T moved into the B-operand layout by movmatrix -- so the
// padded rows cost half as much as in the rows-as-M form and the O
// accumulator needs half the registers (two CTAs per SM).
template <int KS, bool kT, bool kDeep = false>
__global__ void __maxnreg__(kT ? 128 : 255)
    decode_splitkv_kernel(const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const DecodeParams p) {
  using C = DecodeCfg<KS, kDeep>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* ring = smem;
  uint64_t* full = (uint64_t*)(smem + (C::kRingBytes > C::kMergeBytes ? C::kRingBytes
                                                                       : C::kMergeBytes));
  uint64_t* empty = full + C::kStages;
  int* flag = (int*)(empty + C::kStages);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Flattened grid: blockIdx.x = (unit * row_blocks + rb) * splits + split.
  const int split = (int)(blockIdx.x % (unsigned)p.splits);
  const int rb = (int)((blockIdx.x / (unsigned)p.splits) % (unsigned)p.row_blocks);
  const int unit = (int)(blockIdx.x / (unsigned)p.splits / (unsigned)p.row_blocks);
  const long long r0 = (long long)rb * kDecRows;
  const int nr = min(kDecRows, p.rows - (int)r0);
  const MaskSpec ms{p.q_len, p.kv_len, p.causal, p.window};
  const KeyRange kr = key_range_from(ms, r0, nr, kDecTile, p.k_base);
  const int t_begin = split * p.tiles_per_split;
  const int t_end = min(kr.t_count, t_begin + p.tiles_per_split);
  const int n_tiles = max(0, t_end - t_begin);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kDecComputeWarps);
    }
    fence_barrier_init();
    flag[0] = 0;
  }
  __syncthreads();

  if (warp == kDecComputeWarps) {
    // ------------------------------------------------------------ loader
    if (p.app_count > 0 && n_tiles > 0) {
      // New tokens inside this CTA's key tiles go to the caches first (the
      // whole warp), then a proxy fence puts the writes ahead of this
      // warp's TMA loads.  CTAs of other row blocks that load the same
      // tiles write the same bits.
      const int b = (int)(unit / p.kv_heads), h = (int)(unit % p.kv_heads);
      const long long k_lo = (long long)p.k_base + (long long)(kr.t_first + t_begin) * kDecTile;
      const long long k_hi = k_lo + (long long)n_tiles * kDecTile;  // exclusive
      const int d8 = p.head_dim / 8;
      for (int l = 0; l < p.app_count; ++l) {
        const long long j = (long long)p.app_pos + l;
        if (j < k_lo || j >= k_hi) continue;
        const long long slot = p.app_ring ? j % p.app_slots : j;
        const long long dst_row =
            p.app_cache_seq_major ? ((long long)b * p.app_slots + slot) * p.kv_heads + h
                                  : ((long long)b * p.kv_heads + h) * p.app_slots + slot;
        const long long src_row = p.app_new_head_major
                                      ? ((long long)b * p.kv_heads + h) * p.app_count + l
                                      : ((long long)b * p.app_count + l) * p.kv_heads + h;
        for (int c = lane; c < 2 * d8; c += 32) {  // 8 elements per step, keys then values
          const int kv = c >= d8, c8 = kv ? c - d8 : c;
          const long long src = src_row * p.head_dim + 8 * c8;
          uint4 w;
          if (p.app_new_f32) {
            const float4* s4 =
                reinterpret_cast<const float4*>(static_cast<const float*>(kv ? p.app_new_v : p.app_new_k) + src);
            const float4 x0 = s4[0], x1 = s4[1];
            w = make_uint4(pack_bf16(x0.x, x0.y), pack_bf16(x0.z, x0.w), pack_bf16(x1.x, x1.y),
                           pack_bf16(x1.z, x1.w));
          } else {
            w = *reinterpret_cast<const uint4*>(
                static_cast<const __nv_bfloat16*>(kv ? p.app_new_v : p.app_new_k) + src);
          }
          *reinterpret_cast<uint4*>((kv ? p.app_v_cache : p.app_k_cache) +
                                    dst_row * p.head_dim + 8 * c8) = w;
        }
      }
      fence_proxy_async_global();
      __syncwarp();
    }
    if (lane == 0 && n_tiles > 0) {
      tma_prefetch_map(&tm_k);
      tma_prefetch_map(&tm_v);
      const int kvh = (int)(unit % p.kv_heads), bidx = (int)(unit / p.kv_heads);
      int issued = 0;
      for (int t = 0; t < n_tiles; ++t) {
        const int s = t % C::kStages;
        if (t >= C::kStages &&
            !mbar_wait(&empty[s], ((t / C::kStages) - 1) & 1, kStatusTimeoutProducer))
          break;
        uint8_t* kt = ring + s * C::kStageBytes;
        uint8_t* vt = kt + C::kTileBytes;
        const int tv = kr.t_first + t_begin + t;
        // K/V row of the tile: its first key, or its slot tile in a ring.
        const int row0 = p.ring_tiles ? ((p.ring_phase + tv) % p.ring_tiles) * kDecTile
                                      : p.k_base + tv * kDecTile;
        mbar_arrive_expect_tx(&full[s], C::kStageBytes);
#pragma unroll
        for (int c = 0; c < C::kDChunks; ++c) {
          tma_load_4d(kt + c * C::kBoxBytes, &tm_k, &full[s], c * 64, row0, kvh, bidx);
          tma_load_4d(vt + c * C::kBoxBytes, &tm_v, &full[s], c * 64, row0, kvh, bidx);
        }
        ++issued;
      }
      // Never leave with copies in flight: wait for the last loads.
      for (int t = max(0, issued - C::kStages); t < issued; ++t)
        mbar_wait(&full[t % C::kStages], (t / C::kStages) & 1, kStatusTimeoutProducer);
    }
    __syncthreads();  // (A) ring free for the merge scratch
    __syncthreads();  // (B) merge done
    return;
  }

  // -------------------------------------------------------------- compute
  const int wm_count = kT ? 1 : (nr <= 16 ? 1 : (nr <= 32 ? 2 : 4));
  const int wn_count = kDecComputeWarps / wm_count;
  const int D = p.head_dim;
  const int DP = KS * 16;  // padded head dim
  float* mrg = (float*)smem;
  if constexpr (kT) {
    const int wn = warp;  // 16 keys of every 64-key tile
    const int g = lane >> 2, t4 = lane & 3;
    // Q^T fragments (B operand: k = head dim, n = row), straight from global.
    uint32_t qb[KS][2];
    {
      const __nv_bfloat16* qrow = p.q + ((long long)unit * p.rows + r0 + g) * D;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int d = ks * 16 + h * 8 + 2 * t4;
          qb[ks][h] = (g < nr && d < D) ? *(const uint32_t*)(qrow + d) : 0u;
        }
    }
    int lo[2], hi[2];  // rows 2*t4 and 2*t4 + 1
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const long long r = r0 + 2 * t4 + h;
      const int qpos = p.kv_len - p.q_len + (int)(r % p.q_len);
      lo[h] = first_key(ms, qpos);
      hi[h] = last_key(ms, qpos);
    }
    float ot[KS][4];
#pragma unroll
    for (int mt = 0; mt < KS; ++mt) ot[mt][0] = ot[mt][1] = ot[mt][2] = ot[mt][3] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY};
    float l_run[2] = {0.f, 0.f};
    const int mi = lane >> 3, rr = lane & 7;
    for (int t = 0; t < n_tiles; ++t) {
      const int s = t % C::kStages;
      if (!mbar_wait(&full[s], (t / C::kStages) & 1, kStatusTimeoutConsumer)) break;
      const uint32_t kbase = smem_u32(ring + s * C::kStageBytes);
      const uint32_t vbase = kbase + C::kTileBytes;
      const int key0 = p.k_base + (kr.t_first + t_begin + t) * kDecTile;
      const int wkey0 = wn * 16;
      const bool need_mask = !(key0 >= kr.all_lo && key0 + kDecTile - 1 <= kr.all_hi);
      // ---- S^T = K Q^T (16 keys x 8 rows)
      float sc[4] = {0.f, 0.f, 0.f, 0.f};
      {
        const int key = wkey0 + (mi & 1) * 8 + rr;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4(kbase + (ks >> 2) * C::kBoxBytes + sw128(key, (ks * 2 + (mi >> 1)) & 7), a0, a1,
                  a2, a3);
          mma_16816(sc, a0, a1, a2, a3, qb[ks][0], qb[ks][1]);
        }
      }
      // ---- logits: element e is (key g + 8*(e>>1), row 2*t4 + (e&1))
      float x[4];
      bool small = true;
      if (p.use_softcap) {
        const float am = fmaxf(fmaxf(fabsf(sc[0]), fabsf(sc[1])), fmaxf(fabsf(sc[2]), fabsf(sc[3])));
        small = __all_sync(0xffffffffu, am * p.cap_in <= 0.5f);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float v = !p.use_softcap ? sc[e] * p.logit_scale
                  : small        ? p.cap_out * tanh_poly_small(sc[e] * p.cap_in)
                                 : p.cap_out * tanh_fast(sc[e] * p.cap_in);
        if (need_mask) {
          const int j = key0 + wkey0 + g + 8 * (e >> 1);
          if (j < lo[e & 1] || j > hi[e & 1]) v = -INFINITY;
        }
        x[e] = v;
      }
      float base[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float m = fmaxf(x[h], x[h + 2]);
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
        const float m_new = fmaxf(m_run[h], m);
        // Rescale only when the max grew by more than 2^8 (or was -inf).
        if (m_new > m_run[h] + 8.0f || (m_run[h] == -INFINITY && m_new != -INFINITY)) {
          const float alpha = ex2(m_run[h] - m_new);
          m_run[h] = m_new;
          l_run[h] *= alpha;
#pragma unroll
          for (int mt = 0; mt < KS; ++mt) {
            ot[mt][h] *= alpha;
            ot[mt][h + 2] *= alpha;
          }
        }
        base[h] = m_run[h] == -INFINITY ? 0.f : m_run[h];
      }
      float pr[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        pr[e] = ex2(x[e] - base[e & 1]);
        l_run[e & 1] += pr[e];
      }
      const uint32_t b0 = movmatrix_t(pack_bf16(pr[0], pr[1]));
      const uint32_t b1 = movmatrix_t(pack_bf16(pr[2], pr[3]));
      // ---- O^T += V^T P^T (head dim 16 at a time)
      {
        const int key = wkey0 + (mi >> 1) * 8 + rr;
#pragma unroll
        for (int mt = 0; mt < KS; ++mt) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4_t(vbase + (mt >> 2) * C::kBoxBytes + sw128(key, (mt * 2 + (mi & 1)) & 7), a0,
                    a1, a2, a3);
          mma_16816(ot[mt], a0, a1, a2, a3, b0, b1);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    // l is a per-thread partial over its keys: reduce over the 8 lanes of a row.
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 4);
      l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 8);
      l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 16);
    }
    __syncthreads();  // (A) ring drained and no longer read: reuse it as merge scratch
    float* so = mrg + wn * 16 * (DP + 2);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float* row = so + (2 * t4 + h) * (DP + 2);
#pragma unroll
      for (int mt = 0; mt < KS; ++mt) {
        row[mt * 16 + g] = ot[mt][h];
        row[mt * 16 + g + 8] = ot[mt][h + 2];
      }
      if (g == 0) {
        row[DP] = m_run[h];
        row[DP + 1] = l_run[h];
      }
    }
  } else {
  const int wm = warp % wm_count, wn = warp / wm_count;
  const int kw = kDecTile / wn_count;  // keys per warp per tile: 64, 32 or 16
  const int g_row_base = wm * 16 + (lane >> 2);  // CTA row of c0/c1; +8 for c2/c3

  // Q fragments (A operand, row-major 16 x 16 per k-step), straight from global.
  uint32_t qa[KS][4];
  {
    const __nv_bfloat16* qb = p.q + ((long long)unit * p.rows + r0) * D;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const int row = g_row_base + ((h & 1) ? 8 : 0);
        const int d = ks * 16 + ((h & 2) ? 8 : 0) + 2 * (lane & 3);
        uint32_t val = 0;
        if (row < nr && d < D) val = *(const uint32_t*)(qb + (long long)row * D + d);
        qa[ks][h] = val;
      }
    }
  }

  // Per-row mask bounds (rows g_row_base and g_row_base + 8).
  int lo[2], hi[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const long long r = r0 + g_row_base + 8 * h;
    const int qpos = p.kv_len - p.q_len + (int)(r % p.q_len);
    lo[h] = first_key(ms, qpos);
    hi[h] = last_key(ms, qpos);
  }

  float o_acc[2 * KS][4];
#pragma unroll
  for (int n = 0; n < 2 * KS; ++n) o_acc[n][0] = o_acc[n][1] = o_acc[n][2] = o_acc[n][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY};
  float l_run[2] = {0.f, 0.f};
  bool ok = true;

  for (int t = 0; t < n_tiles && ok; ++t) {
    const int s = t % C::kStages;
    if (!mbar_wait(&full[s], (t / C::kStages) & 1, kStatusTimeoutConsumer)) {
      ok = false;
      break;
    }
    const uint32_t kbase = smem_u32(ring + s * C::kStageBytes);
    const uint32_t vbase = kbase + C::kTileBytes;
    const int key0 = p.k_base + (kr.t_first + t_begin + t) * kDecTile;
    const int wkey0 = wn * kw;  // first key of this warp inside the tile
    const bool need_mask = !(key0 >= kr.all_lo && key0 + kDecTile - 1 <= kr.all_hi);

    for (int kk = 0; kk < kw / 16; ++kk) {
      // ---- S = Q K^T for 16 keys (two n8 tiles)
      float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      {
        const int mi = lane >> 3, rr = lane & 7;
        const int key = wkey0 + kk * 16 + (mi >> 1) * 8 + rr;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          const int chunk = (ks * 2 + (mi & 1)) & 7;
          const int box = (ks * 16) / 64;
          uint32_t b0, b1, b2, b3;
          ldsm_x4(kbase + box * C::kBoxBytes + sw128(key, chunk), b0, b1, b2, b3);
          mma_16816(sc[0], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b0, b1);
          mma_16816(sc[1], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b2, b3);
        }
      }
      // ---- logits (log2 domain), softcap, mask.  With a softcap the tanh is
      // an FMA-pipe polynomial when every |x / s| of the warp is <= 1/2.
      float x[2][4];
      if (p.use_softcap) {
        float am = 0.f;
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e) am = fmaxf(am, fabsf(sc[n][e]));
        if (__all_sync(0xffffffffu, am * p.cap_in <= 0.5f)) {
#pragma unroll
          for (int n = 0; n < 2; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) x[n][e] = p.cap_out * tanh_poly_small(sc[n][e] * p.cap_in);
        } else {
#pragma unroll
          for (int n = 0; n < 2; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) x[n][e] = p.cap_out * tanh_fast(sc[n][e] * p.cap_in);
        }
      } else {
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e) x[n][e] = sc[n][e] * p.logit_scale;
      }
      if (need_mask) {
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int j = key0 + wkey0 + kk * 16 + n * 8 + 2 * (lane & 3) + (e & 1);
            const int h = e >> 1;
            if (j < lo[h] || j > hi[h]) x[n][e] = -INFINITY;
          }
      }
      // ---- online softmax update (two rows per thread, quad-wide max);
      // O is rescaled only when a row max grows by more than 2^8.
      float base[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float m = fmaxf(fmaxf(x[0][2 * h], x[0][2 * h + 1]), fmaxf(x[1][2 * h], x[1][2 * h + 1]));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
        const float m_new = fmaxf(m_run[h], m);
        if (m_new > m_run[h] + 8.0f || (m_run[h] == -INFINITY && m_new != -INFINITY)) {
          const float alpha = ex2(m_run[h] - m_new);  // 0 when m_run = -inf
          m_run[h] = m_new;
          l_run[h] *= alpha;
#pragma unroll
          for (int n = 0; n < 2 * KS; ++n) {
            o_acc[n][2 * h] *= alpha;
            o_acc[n][2 * h + 1] *= alpha;
          }
        }
        base[h] = (m_run[h] == -INFINITY) ? 0.f : m_run[h];
      }
      float pr[2][4];
#pragma unroll
      for (int n = 0; n < 2; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          pr[n][e] = ex2(x[n][e] - base[e >> 1]);
          l_run[e >> 1] += pr[n][e];
        }
      const uint32_t a0 = pack_bf16(pr[0][0], pr[0][1]);
      const uint32_t a1 = pack_bf16(pr[0][2], pr[0][3]);
      const uint32_t a2 = pack_bf16(pr[1][0], pr[1][1]);
      const uint32_t a3 = pack_bf16(pr[1][2], pr[1][3]);
      // ---- O += P V for these 16 keys
      {
        const int mi = lane >> 3, rr = lane & 7;
        const int key = wkey0 + kk * 16 + (mi & 1) * 8 + rr;
#pragma unroll
        for (int dn = 0; dn < KS; ++dn) {
          const int chunk = (dn * 2 + (mi >> 1)) & 7;
          const int box = (dn * 16) / 64;
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(vbase + box * C::kBoxBytes + sw128(key, chunk), b0, b1, b2, b3);
          mma_16816(o_acc[2 * dn], a0, a1, a2, a3, b0, b1);
          mma_16816(o_acc[2 * dn + 1], a0, a1, a2, a3, b2, b3);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }

  // l is per-thread partial over its columns: reduce across the quad.
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 1);
    l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 2);
  }

  // ---- merge the key-slices of the warps through shared memory
  __syncthreads();  // (A) ring drained and no longer read: reuse it as merge scratch
  {
    const int slot = wn * wm_count + wm;  // 0..3
    float* so = mrg + slot * 16 * (DP + 2);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = (lane >> 2) + 8 * h;
      float* row = so + r * (DP + 2);
#pragma unroll
      for (int n = 0; n < 2 * KS; ++n) {
        row[n * 8 + 2 * (lane & 3)] = o_acc[n][2 * h];
        row[n * 8 + 2 * (lane & 3) + 1] = o_acc[n][2 * h + 1];
      }
      if ((lane & 3) == 0) {
        row[DP] = m_run[h];
        row[DP + 1] = l_run[h];
      }
    }
  }
  }
  asm volatile("bar.sync 1, %0;" ::"r"(kDecComputeWarps * 32) : "memory");

  const bool direct = p.splits == 1;
  const long long prow0 = (((long long)unit * p.row_blocks + rb) * p.splits + split) * p.block_rows;
  for (int idx = threadIdx.x; idx < nr * D; idx += kDecComputeWarps * 32) {
    const int row = idx / D, d = idx - (idx / D) * D;
    const int rwm = row >> 4, r = row & 15;
    float M = -INFINITY;
    for (int w = 0; w < wn_count; ++w)
      M = fmaxf(M, mrg[((w * wm_count + rwm) * 16 + r) * (DP + 2) + DP]);
    const float Mb = (M == -INFINITY) ? 0.f : M;
    float L = 0.f, O = 0.f;
    for (int w = 0; w < wn_count; ++w) {
      const float* row_p = mrg + ((w * wm_count + rwm) * 16 + r) * (DP + 2);
      const float f = ex2(row_p[DP] - Mb);
      L += f * row_p[DP + 1];
      O += f * row_p[d];
    }
    const float o_val = L > 0.f ? O / L : 0.f;
    if (direct) {
      p.o[((long long)unit * p.rows + r0 + row) * D + d] = __float2bfloat16_rn(o_val);
    } else {
      p.part_o[(prow0 + row) * D + d] = o_val;
      if (d == 0) p.part_lse[prow0 + row] = L > 0.f ? M + log2f(L) : -INFINITY;
    }
  }
  __syncthreads();  // (B) pairs with the loader's second barrier
  if (direct) return;

  // ---- last CTA of this row block merges the split partials
  __threadfence();
  asm volatile("bar.sync 1, %0;" ::"r"(kDecComputeWarps * 32) : "memory");
  if (threadIdx.x == 0) {
    const unsigned int ticket = atomicAdd(&p.tickets[unit * p.row_blocks + rb], 1u);
    flag[0] = (ticket == (unsigned)p.splits - 1) ? 1 : 0;
  }
  asm volatile("bar.sync 1, %0;" ::"r"(kDecComputeWarps * 32) : "memory");
  if (!flag[0]) return;
  __threadfence();
  // Split weights w_s = 2^(lse_s - M) / sum_s 2^(lse_s - M) per row, in the
  // (now idle) ring; then every thread streams float4 chunks of the partials
  // with independent loads.
  const long long pbase = ((long long)unit * p.row_blocks + rb) * p.splits * p.block_rows;
  float* wgt = (float*)smem;  // [split][nr]
  for (int row = threadIdx.x; row < nr; row += kDecComputeWarps * 32) {
    float M = -INFINITY;
    for (int s = 0; s < p.splits; ++s)
      M = fmaxf(M, __ldcg(&p.part_lse[pbase + (long long)s * p.block_rows + row]));
    float L = 0.f;
    for (int s = 0; s < p.splits; ++s) {
      const float f = M == -INFINITY
                          ? 0.f
                          : ex2(__ldcg(&p.part_lse[pbase + (long long)s * p.block_rows + row]) - M);
      wgt[s * nr + row] = f;
      L += f;
    }
    const float inv = L > 0.f ? 1.0f / L : 0.f;
    for (int s = 0; s < p.splits; ++s) wgt[s * nr + row] *= inv;
  }
  asm volatile("bar.sync 1, %0;" ::"r"(kDecComputeWarps * 32) : "memory");
  const int d4 = D / 4;
  for (int idx = threadIdx.x; idx < nr * d4; idx += kDecComputeWarps * 32) {
    const int row = idx / d4, c = idx - (idx / d4) * d4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int s = 0; s < p.splits; ++s) {
      const float w = wgt[s * nr + row];
      const float4 v = __ldcg(reinterpret_cast<const float4*>(
          p.part_o + (pbase + (long long)s * p.block_rows + row) * D) + c);
      acc.x += w * v.x;
      acc.y += w * v.y;
      acc.z += w * v.z;
      acc.w += w * v.w;
    }
    uint2 packed = make_uint2(pack_bf16(acc.x, acc.y), pack_bf16(acc.z, acc.w));
    *reinterpret_cast<uint2*>(p.o + ((long long)unit * p.rows + r0 + row) * D + 4 * c) = packed;
  }
  if (threadIdx.x == 0) p.tickets[unit * p.row_blocks + rb] = 0u;  // ready for the next call
}

}  // namespace gqa
