// prefill_sm100.cuh -- masked GQA attention for long query blocks (prefill
// and encoder shapes) on the 5th-generation tensor cores of sm_100a.
//
// Rows: for one (batch b, kv head) unit, the R = group * q_len q rows of all
// q heads of the GQA group, in memory order (head-major, then position), are
// cut into 128-row tiles.  A CTA owns two tiles whose key ranges coincide or
// overlap (two heads of the group at the same positions when q_len is a
// multiple of 128, else two consecutive tiles), so every K/V tile it loads
// feeds both ("north star" (2): the q heads of a GQA group are packed so each
// K/V tile is read once).
//
// Roles (12 warps, three warpgroups):
//   warp 0      TMA loader: both Q tiles once, then K_j, V_j (128 keys x
//               head_dim, 128-byte swizzle) into a ring of shared-memory
//               slots guarded by mbarriers;
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer:
//               S_t = Q_t K_j^T (M=128, N=128, fp32 in TMEM) and
//               O_t += P_t V_j (A = P from TMEM, B = V from shared memory,
//               N = head_dim rounded up to 16);
//   warps 2-3   idle (they complete warpgroup 0 for the register split);
//   warps 4-7   softmax + epilogue for tile A, warps 8-11 for tile B: one
//               thread per row reads its S row from TMEM, applies scale,
//               softcap and mask, keeps the running max / sum in fp32
//               (online softmax, rescaling O in TMEM only when the max grows
//               by more than 2^8), writes P as bf16 back over S in TMEM, and
//               at the end normalises O and stores bf16 rows of o.
// The issue order S_A(j+1) after PV_A(j), S_B(j+1) after PV_B(j) keeps the
// tensor pipe busy with one tile while the other tile's softmax runs.
//
// Fully masked key tiles are never loaded; tiles wholly inside every row's
// visible range skip the per-element mask.  All waits are bounded.
#pragma once

#include "mask.cuh"
#include "ptx.cuh"

namespace gqa {

constexpr int kPfM = 128;       // rows per q tile
constexpr int kPfN = 128;       // keys per K/V tile
constexpr int kPfWarps = 12;
constexpr int kPfThreads = 32 * kPfWarps;
// Register split (setmaxnreg): the loader/MMA warpgroup drops to kRegsLow,
// the two softmax warpgroups rise to kRegsHigh.  The host checks before every
// launch that 4*32*kRegsLow + 8*32*kRegsHigh fits in the registers the block
// is launched with, so the increase can always be granted.
constexpr int kRegsLow = 96;
constexpr int kRegsHigh = 200;
constexpr int kRegSplitTotal = 4 * 32 * kRegsLow + 8 * 32 * kRegsHigh;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct PrefillParams {
  __nv_bfloat16* o;
  int q_len, kv_len, head_dim, d_pad;
  int rows;              // rows per unit: group * q_len
  int tiles_per_unit;    // ceil(rows / 128)
  int pairs_per_unit;    // CTAs per unit
  int pair_heads;        // 1: tiles (2p, 2p+1) are two heads at one position
  int causal, window;
  int use_softcap;
  float logit_scale, cap_in, cap_out;
};

template <int DCH>
struct PrefillCfg {
  static constexpr int kBoxBytes = 128 * 128;            // 128 rows x 64 bf16
  static constexpr int kTileBytes = DCH * kBoxBytes;     // one Q, K or V tile
  static constexpr int kSlots = DCH == 1 ? 8 : 4;
  static constexpr int kQBytes = 2 * kTileBytes;
  static constexpr int kRingBytes = kSlots * kTileBytes;
  static constexpr int kBarOffset = kQBytes + kRingBytes;
  // barriers: q_full, kv_full[S], kv_empty[S], s_full[2], p_full[2], o_done[2], drain
  static constexpr int kNumBars = 1 + 2 * kSlots + 2 + 2 + 2 + 1;
  static constexpr int kSmemBytes = 1024 + kBarOffset + kNumBars * 8 + 16;
};

struct TileInfo {
  int row0;       // first row of the tile in the unit's row block
  int nrows;      // valid rows (0 = no tile)
  KeyRange kr;    // key tiles this tile touches
};

__device__ __forceinline__ TileInfo prefill_tile(const PrefillParams& p, const MaskSpec& ms,
                                                 int pair, int which) {
  TileInfo ti;
  int tile;
  if (p.pair_heads) {
    const int tiles_per_head = p.q_len / kPfM;
    const int pos = pair % tiles_per_head, hp = pair / tiles_per_head;
    tile = (2 * hp + which) * tiles_per_head + pos;
  } else {
    tile = 2 * pair + which;
  }
  ti.row0 = tile * kPfM;
  ti.nrows = tile < p.tiles_per_unit ? min(kPfM, p.rows - ti.row0) : 0;
  if (ti.nrows > 0) {
    ti.kr = key_range(ms, ti.row0, ti.nrows, kPfN);
  } else {
    ti.kr.t_first = 0;
    ti.kr.t_count = 0;
    ti.kr.all_lo = 1;
    ti.kr.all_hi = 0;
  }
  return ti;
}

template <int DCH>
__global__ void __launch_bounds__(kPfThreads, 1)
    prefill_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const PrefillParams p) {
  using C = PrefillCfg<DCH>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sq = smem;                   // Q tiles A, B
  uint8_t* ring = smem + C::kQBytes;    // K/V slots
  uint64_t* bars = (uint64_t*)(smem + C::kBarOffset);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + C::kSlots;
  uint64_t* s_full = kv_empty + C::kSlots;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_done = p_full + 2;
  uint64_t* drain = o_done + 2;
  uint32_t* tmem_slot = (uint32_t*)(drain + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int unit = blockIdx.x / p.pairs_per_unit;
  const int pair = blockIdx.x % p.pairs_per_unit;
  const MaskSpec ms{p.q_len, p.kv_len, p.causal, p.window};
  const TileInfo ta = prefill_tile(p, ms, pair, 0);
  const TileInfo tb = prefill_tile(p, ms, pair, 1);
  // Key tiles of the CTA: the union of both tiles' ranges.
  int j_first, j_count;
  {
    const bool ea = ta.kr.t_count == 0, eb = tb.kr.t_count == 0;
    if (ea && eb) {
      j_first = 0;
      j_count = 0;
    } else {
      const int fa = ea ? 0x7fffffff : ta.kr.t_first, fb = eb ? 0x7fffffff : tb.kr.t_first;
      const int la = ea ? -1 : ta.kr.t_first + ta.kr.t_count - 1;
      const int lb = eb ? -1 : tb.kr.t_first + tb.kr.t_count - 1;
      j_first = min(fa, fb);
      j_count = max(la, lb) - j_first + 1;
    }
  }

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < C::kSlots; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 128);
      mbar_init(&o_done[t], 1);
    }
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // TMEM columns: S_A [0,128), S_B [128,256), O_A [256,384), O_B [384,512).
  // P_t (bf16 pairs) overwrites the first 64 columns of S_t.

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow));
  }
  if (warp == 0) {
    // ------------------------------------------------------------ loader
    if (lane == 0) {
      tma_prefetch_map(&tm_q);
      tma_prefetch_map(&tm_k);
      tma_prefetch_map(&tm_v);
      const int nq = (ta.nrows > 0 ? 1 : 0) + (tb.nrows > 0 ? 1 : 0);
      if (nq > 0 && j_count > 0) {
        mbar_arrive_expect_tx(q_full, nq * C::kTileBytes);
        for (int c = 0; c < DCH; ++c) {
          if (ta.nrows > 0)
            tma_load_3d(sq + c * C::kBoxBytes, &tm_q, q_full, c * 64, ta.row0, unit);
          if (tb.nrows > 0)
            tma_load_3d(sq + C::kTileBytes + c * C::kBoxBytes, &tm_q, q_full, c * 64, tb.row0,
                        unit);
        }
      }
      int issued = 0;
      bool ok = true;
      for (int j = 0; j < j_count && ok; ++j) {
        const int key0 = (j_first + j) * kPfN;
        for (int kv = 0; kv < 2; ++kv) {
          const int u = 2 * j + kv;
          const int s = u % C::kSlots;
          if (u >= C::kSlots &&
              !mbar_wait(&kv_empty[s], ((u / C::kSlots) - 1) & 1, kStatusTimeoutProducer)) {
            ok = false;
            break;
          }
          uint8_t* dst = ring + s * C::kTileBytes;
          mbar_arrive_expect_tx(&kv_full[s], C::kTileBytes);
          for (int c = 0; c < DCH; ++c)
            tma_load_3d(dst + c * C::kBoxBytes, kv ? &tm_v : &tm_k, &kv_full[s], c * 64, key0,
                        unit);
          ++issued;
        }
      }
      // Drain: never leave with copies in flight.
      if (nq > 0 && j_count > 0) mbar_wait(q_full, 0, kStatusTimeoutProducer);
      for (int u = max(0, issued - C::kSlots); u < issued; ++u)
        mbar_wait(&kv_full[u % C::kSlots], (u / C::kSlots) & 1, kStatusTimeoutProducer);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && j_count > 0) {
      const uint32_t idesc_s = idesc_bf16_f32(kPfM, kPfN, 0);
      const uint32_t idesc_o = idesc_bf16_f32(kPfM, p.d_pad, 1);
      const int ksteps = p.d_pad / 16;
      const uint32_t sq_addr = smem_u32(sq);
      const uint32_t ring_addr = smem_u32(ring);
      int n_act[2] = {0, 0};
      bool ok = mbar_wait(q_full, 0, kStatusTimeoutMma);

      auto active = [&](int t, int j) {
        const KeyRange& kr = t == 0 ? ta.kr : tb.kr;
        const int jj = j_first + j;
        return kr.t_count > 0 && jj >= kr.t_first && jj < kr.t_first + kr.t_count;
      };
      auto wait_slot = [&](int u) {
        return mbar_wait(&kv_full[u % C::kSlots], (u / C::kSlots) & 1, kStatusTimeoutMma);
      };
      auto issue_s = [&](int t, int j) {
        const uint32_t kslot = ring_addr + ((2 * j) % C::kSlots) * C::kTileBytes;
        const uint32_t qt = sq_addr + t * C::kTileBytes;
        const uint32_t d_tmem = tmem + t * 128;
        tc_fence_after();
        for (int ks = 0; ks < ksteps; ++ks) {
          const uint32_t off = (ks >> 2) * C::kBoxBytes + (ks & 3) * 32;
          mma_bf16_ss(d_tmem, sdesc_sw128(qt + off, 16, 1024), sdesc_sw128(kslot + off, 16, 1024),
                      idesc_s, ks > 0 ? 1u : 0u);
        }
        mma_commit(&s_full[t]);
      };
      auto issue_pv = [&](int t, int j) {
        const uint32_t vslot = ring_addr + ((2 * j + 1) % C::kSlots) * C::kTileBytes;
        const uint32_t p_tmem = tmem + t * 128;
        const uint32_t o_tmem = tmem + 256 + t * 128;
        tc_fence_after();
        for (int ks = 0; ks < kPfN / 16; ++ks) {
          mma_bf16_ts(o_tmem, p_tmem + ks * 8, sdesc_sw128(vslot + ks * 2048, C::kBoxBytes, 1024),
                      idesc_o, (n_act[t] > 0 || ks > 0) ? 1u : 0u);
        }
      };

      // Prologue: S(0) for both tiles.
      if (ok) ok = wait_slot(0);
      for (int t = 0; t < 2 && ok; ++t)
        if (active(t, 0)) issue_s(t, 0);
      for (int j = 0; j < j_count && ok; ++j) {
        if (!(ok = wait_slot(2 * j + 1))) break;  // V_j
        bool k_next_ready = j + 1 >= j_count;
        for (int t = 0; t < 2 && ok; ++t) {
          if (active(t, j)) {
            if (!(ok = mbar_wait(&p_full[t], n_act[t] & 1, kStatusTimeoutMma))) break;
            issue_pv(t, j);
            ++n_act[t];
          }
          if (j + 1 < j_count && active(t, j + 1)) {
            if (!k_next_ready) {
              if (!(ok = wait_slot(2 * (j + 1)))) break;  // K_{j+1}
              k_next_ready = true;
            }
            issue_s(t, j + 1);
          }
        }
        // K_{j+1} must have landed before iteration j+1 can release it.
        if (ok && !k_next_ready) ok = wait_slot(2 * (j + 1));
        if (!ok) break;
        // Release K_j and V_j once everything issued so far has completed.
        mma_commit(&kv_empty[(2 * j) % C::kSlots]);
        mma_commit(&kv_empty[(2 * j + 1) % C::kSlots]);
      }
      mma_commit(&o_done[0]);
      mma_commit(&o_done[1]);
      // Drain: every MMA finished before TMEM can be released.
      mma_commit(drain);
      mbar_wait(drain, 0, kStatusTimeoutMma);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax / epilogue
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsHigh));
    const int t = (warp - 4) / 4;            // tile 0 (A) or 1 (B)
    const TileInfo& ti = t == 0 ? ta : tb;
    const int quarter = warp & 3;            // TMEM lane quarter of this warp
    const int r = quarter * 32 + lane;       // row within the tile
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const uint32_t s_tmem = tmem + lane_base + t * 128;
    const uint32_t o_tmem = tmem + lane_base + 256 + t * 128;
    const long long grow = (long long)ti.row0 + r;  // row within the unit
    const bool row_valid = r < ti.nrows;
    int lo = 0, hi = -1;
    if (row_valid) {
      const int qpos = p.kv_len - p.q_len + (int)(grow % p.q_len);
      lo = first_key(ms, qpos);
      hi = last_key(ms, qpos);
    }
    float m_run = -INFINITY, l_run = 0.f;
    int n_act = 0;
    bool ok = true;
    for (int j = 0; j < j_count && ok; ++j) {
      const int jj = j_first + j;
      if (ti.kr.t_count == 0 || jj < ti.kr.t_first || jj >= ti.kr.t_first + ti.kr.t_count)
        continue;
      ok = __all_sync(0xffffffffu, mbar_wait(&s_full[t], n_act & 1, kStatusTimeoutSoftmax));
      if (!ok) break;
      tc_fence_after();
      uint32_t s0[32], s1[32], s2[32], s3[32];
      tmem_ld32(s_tmem + 0, s0);
      tmem_ld32(s_tmem + 32, s1);
      tmem_ld32(s_tmem + 64, s2);
      tmem_ld32(s_tmem + 96, s3);
      tmem_ld_wait();
      float x[128];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        x[c] = __uint_as_float(s0[c]);
        x[32 + c] = __uint_as_float(s1[c]);
        x[64 + c] = __uint_as_float(s2[c]);
        x[96 + c] = __uint_as_float(s3[c]);
      }
      const int key0 = jj * kPfN;
      const bool need_mask = !(key0 >= ti.kr.all_lo && key0 + kPfN - 1 <= ti.kr.all_hi);
      if (p.use_softcap) {
#pragma unroll
        for (int c = 0; c < 128; ++c) x[c] = p.cap_out * tanh_accurate(x[c] * p.cap_in);
      } else {
#pragma unroll
        for (int c = 0; c < 128; ++c) x[c] *= p.logit_scale;
      }
      if (need_mask) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (key0 + c < lo || key0 + c > hi) x[c] = -INFINITY;
      }
      float mt = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; ++c) mt = fmaxf(mt, x[c]);
      // Rescale only when the max grew by more than 2^8 (or was -inf): the
      // stale max keeps p <= 256, and O / l stays consistent either way.
      const float m_new = fmaxf(m_run, mt);
      const bool need =
          (m_new > m_run + kRescaleThreshold) || (m_run == -INFINITY && m_new != -INFINITY);
      const float alpha = need ? ex2(m_run - m_new) : 1.0f;  // 0 when m_run = -inf
      if (need) {
        l_run *= alpha;
        m_run = m_new;
      }
      if (__any_sync(0xffffffffu, need) && n_act > 0) {
        // tcgen05.ld/st are warp-collective: every lane takes part.
        for (int c0 = 0; c0 < p.d_pad; c0 += 16) {
          uint32_t ov[16];
          tmem_ld16(o_tmem + c0, ov);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 16; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
          tmem_st16(o_tmem + c0, ov);
        }
        tmem_st_wait();
      }
      const float base = m_run == -INFINITY ? 0.f : m_run;
      float ls = 0.f;
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const float p0 = ex2(x[32 * q4 + 2 * c] - base);
          const float p1 = ex2(x[32 * q4 + 2 * c + 1] - base);
          ls += p0 + p1;
          pk[c] = pack_bf16(p0, p1);
        }
        tmem_st16(s_tmem + 16 * q4, pk);
      }
      l_run += ls;
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[t]);
      ++n_act;
    }
    // ---- epilogue: o = O / l, bf16, one row per thread (warp-collective loads)
    if (__all_sync(0xffffffffu, ok) && ti.nrows > 0) {
      const bool have = n_act > 0;
      bool ready = true;
      if (have) {
        ready = __all_sync(0xffffffffu, mbar_wait(&o_done[t], 0, kStatusTimeoutEpilogue));
        tc_fence_after();
      }
      if (ready) {
        const bool live = have && l_run > 0.f;
        const float inv = live ? 1.0f / l_run : 0.f;
        __nv_bfloat16* orow = p.o + ((long long)unit * p.rows + grow) * p.head_dim;
        for (int c0 = 0; c0 < p.head_dim; c0 += 16) {
          uint32_t ov[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) ov[e] = 0u;
          if (have) {
            tmem_ld16(o_tmem + c0, ov);
            tmem_ld_wait();
          }
          uint32_t w[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float a = live ? __uint_as_float(ov[2 * e]) * inv : 0.f;
            const float b = live ? __uint_as_float(ov[2 * e + 1]) * inv : 0.f;
            w[e] = pack_bf16(a, b);
          }
          if (row_valid) {
            uint4* dst = reinterpret_cast<uint4*>(orow + c0);
            dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
            if (c0 + 16 <= p.head_dim) dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
          }
        }
      }
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace gqa
