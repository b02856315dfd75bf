// prefill_sm100.cuh -- masked GQA attention for long query blocks (prefill
// and encoder shapes) on the 5th-generation tensor cores of sm_100a.
//
// Rows: for one (batch b, kv head) unit, the R = group * q_len q rows of all
// q heads of the GQA group, in memory order (head-major, then position), are
// cut into 128-row tiles.  A work item is a pair of tiles whose key ranges
// coincide or overlap (two heads of the group at the same positions when
// q_len is a multiple of 128, else two consecutive tiles), so every K/V tile
// loaded for the item feeds both: the q heads of a GQA group share one kv
// head ("TPU v6e Masked GQA Kernel Optimization", "What You Have": GQA
// ratios 1:1 to 16:1), so its K/V tiles are read once for all of them.
//
// Persistent: one CTA per SM walks one item per round of gridDim.x items
// (blockIdx.x of each round, or its mirror image on odd rounds when the items
// are sorted heavy first: snake_item); TMEM, barriers and the K/V ring live
// across items, and the
// next item's Q is loaded as soon as the current item's last S = Q K^T has
// been computed, so loads, MMAs and softmax of consecutive items overlap.
//
// Roles (12 warps, three warpgroups):
//   warp 0      TMA loader: Q tiles, then K_j, V_j (128 keys x head_dim,
//               128-byte swizzle) into a ring of shared-memory slots guarded
//               by mbarriers (for paired items, below, K only: warp 2
//               streams V through its own half of the ring);
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer:
//               S_t = Q_t K_j^T (M=128, N=128, fp32 in TMEM) and
//               O_t += P_t V_j (A = P from TMEM, B = V from shared memory,
//               N = head_dim rounded up to 16);
//   warps 2-3   idle but for warp 2's V stream of paired items (they
//               complete warpgroup 0 for the register split);
//   warps 4-7   softmax + epilogue of q tile A, warps 8-11 of q tile B: a
//               thread owns one row of its tile.  It reads the row's 128
//               scores of an S tile from TMEM, applies scale, softcap and
//               mask, keeps the running max and sum in fp32 (online softmax,
//               rescaling its O row in TMEM only when the max grows by more
//               than 2^8), writes P as bf16 back over S in TMEM, and at the
//               end of the item normalises its O row and stores it.  P.V is
//               handed over in two halves: keys 0..63 (p_half) while the
//               softmax still works on keys 64..127 (p_full).  With a
//               softcap the logits are bounded, so caps up to about 63.8 use
//               a fixed exponent base and one pass over the scores, with no
//               row max and no rescale (PrefillParams::cap_fixed).
// The two softmax warpgroups work on their own tiles at the same time, out
// of phase: while one computes its softmax the tensor core runs the other
// tile's P.V and next S, and the two warps each SM sub-partition holds (one
// per tile) hide each other's waits.  The MMA thread serves tile A, then
// tile B, which keeps them half a step apart; serving events as they come,
// or making the warpgroups take turns, was measured slower.  The softmax
// code is one compact path for every tile (masked tiles get -inf written
// over their hidden scores first): separate unrolled copies for masked
// tiles missed the instruction cache each time they ran.
//
// Fully masked key tiles are never loaded; tiles wholly inside every row's
// visible range skip the per-element mask.  All waits are bounded.
#pragma once

#include <type_traits>

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
constexpr int kRegsLow = 120;
constexpr int kRegsHigh = 192;
constexpr int kRegSplitTotal = 4 * 32 * kRegsLow + 8 * 32 * kRegsHigh;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// Without a softcap, pairs [kEmuFrom, 16) of every 16 score pairs (32 keys)
// of a row take 2^x from exp2_poly_x2 (FMA pipe), the rest from MUFU.
// Measured on B200: one pair in eight was 2-3% faster on the encoder shape;
// a quarter or a half was slower.  The softcap kernels already spend FMA
// work on the tanh polynomial and keep every 2^x on MUFU.
constexpr int kEmuFrom = 14;

struct PrefillParams {
  __nv_bfloat16* o;
  int q_len, kv_len, head_dim, d_pad;
  int kv_heads;          // K/V maps are 4-D: (col, key, kv head, batch)
  int rows;              // rows per unit: group * q_len
  int tiles_per_unit;    // ceil(rows / 128)
  int pairs_per_unit;    // tile pairs per unit (row tiles per unit when split_pairs)
  int splits;            // key-range splits per tile pair (1 = none)
  int split_pairs;       // 1: both tiles of an item are the same row tile, taking
                         // key splits 2s and 2s + 1 (units with one row tile)
  int n_items;           // units * pairs_per_unit * splits (/ 2 when split_pairs)
  int pair_heads;        // 1: tiles (2p, 2p+1) are two heads at one position
  int heavy_first;       // 1: items run in order of decreasing key-tile count (causal / window)
  int cluster_merge;     // paired items, one per CTA, launched as clusters of this many CTAs
                         // (one cluster per unit): after one cluster barrier every CTA
                         // merges a column slice of the unit's partials from the
                         // workspace; 0 = the last CTA of a unit merges (tickets)
  int causal, window;
  float logit_scale, cap_in, cap_out;
  // Softcap with a fixed exponent base (cap_fixed = 1, softcap code 3): the capped logits,
  // in log2 units, lie in [-cap_out, cap_out], so p = 2^(y - cap_base) with
  // cap_base = cap_out - B stays in [2^(B - 2 cap_out), 2^B].  The host picks
  // B = max(16, 2 cap_out - 120) and sets cap_fixed only when B <= 64, so p
  // never overflows or leaves the normal range and no row max is needed.
  int cap_fixed;
  float cap_base;
  // Split partials (splits > 1): per (pair, tile, split) O as fp32
  // [d / 4][128 rows][4] (a thread moves four columns of its row as one
  // 16-byte access and a warp's accesses coalesce) and (m, l) per row;
  // tickets per (pair, tile, warp) count the splits that have finished.
  float* ws_o;
  float* ws_ml;
  unsigned int* tickets;
};

template <int DCH>
struct PrefillCfg {
  static constexpr int kBoxBytes = 128 * 128;            // 128 rows x 64 bf16
  static constexpr int kTileBytes = DCH * kBoxBytes;     // one Q, K or V tile
  static constexpr int kSlots = DCH == 1 ? 8 : 4;
  static constexpr int kQBytes = 2 * kTileBytes;
  static constexpr int kRingBytes = kSlots * kTileBytes;
  // Output staging: one 32-row x 64-column bf16 box (4 KB) per softmax warp.
  static constexpr int kStageBytes = 8 * 4096;
  // (m, l) of a row swapped between the two softmax warpgroups (paired key
  // splits, which write no output through the staging boxes):
  // [warpgroup][row] float2 at this offset in the staging area.
  static constexpr int kXchgOffset = 16384;
  static constexpr int kBarOffset = kQBytes + kRingBytes + kStageBytes;
  // q_full, q_empty, kv_full[S], kv_empty[S], s_full[2], p_full[2], o_done[2],
  // drain, part_done[2], flag_ready[2], p_half[2]
  static constexpr int kNumBars = 2 + 2 * kSlots + 2 + 2 + 2 + 1 + 2 + 2 + 2;
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

// One work item: a unit, its pair of q tiles and one split of the union of
// their key-tile ranges: key tiles [j_first, j_first + j_count).  With
// split_pairs both tiles are the same row tile and take adjacent key splits:
// tile t processes key tiles [kt0[t], kt0[t] + kc[t]), so the two softmax
// warpgroups still alternate.  An item without key tiles is not "busy": no
// loads or MMAs run for it.
struct PfItem {
  int unit;
  int pair_index;  // unit * pairs_per_unit + pair
  int split;       // split of tile 0 (tile 1 takes split + 1 when paired)
  bool paired;
  TileInfo tile[2];
  int j_first, j_count;
  int kt0[2], kc[2];
  bool busy;
};

template <int kSplit>
__device__ __forceinline__ PfItem prefill_item(const PrefillParams& p, const MaskSpec& ms,
                                               int item) {
  PfItem it;
  it.paired = kSplit == 2 || (kSplit == 1 && p.split_pairs != 0);
  if (it.paired) {
    const int half = p.splits / 2;
    it.split = 2 * (item % half);
    it.pair_index = item / half;
    it.unit = it.pair_index / p.pairs_per_unit;
    const int tile = it.pair_index % p.pairs_per_unit;
    TileInfo ti;
    ti.row0 = tile * kPfM;
    ti.nrows = min(kPfM, p.rows - ti.row0);
    ti.kr = key_range(ms, ti.row0, ti.nrows, kPfN);
    it.tile[0] = ti;
    it.tile[1] = ti;
    // Split s takes key tiles [ceil(s T / S), ceil((s + 1) T / S)): sizes
    // differ by at most one.  Tile A takes the larger of the item's two.
    const int T = ti.kr.t_count, S = p.splits;
    for (int t = 0; t < 2; ++t) {
      const int sp = it.split + t;
      const int js = (sp * T + S - 1) / S, je = ((sp + 1) * T + S - 1) / S;
      it.kt0[t] = ti.kr.t_first + js;
      it.kc[t] = je - js;
    }
    if (it.kc[1] > it.kc[0]) {
      const int k0 = it.kt0[0], c0 = it.kc[0];
      it.kt0[0] = it.kt0[1];
      it.kc[0] = it.kc[1];
      it.kt0[1] = k0;
      it.kc[1] = c0;
    }
    it.j_first = it.kt0[0];
    it.j_count = it.kc[0];  // kc[0] >= kc[1]
    it.busy = it.j_count > 0;
    return it;
  }
  it.split = item % p.splits;
  it.pair_index = item / p.splits;
  int pair;
  if (p.heavy_first) {
    // Causal / windowed rows see more keys the later their position (up to
    // the window): walk positions from the last down, all units at each
    // rank, so the CTAs' last rounds hold the lightest items.
    const int units = p.n_items / (p.splits * p.pairs_per_unit);
    const int rank = it.pair_index / units;
    it.unit = it.pair_index % units;
    if (p.pair_heads) {
      const int tiles_per_head = p.q_len / kPfM;
      const int n_hp = p.pairs_per_unit / tiles_per_head;
      pair = (rank % n_hp) * tiles_per_head + (tiles_per_head - 1 - rank / n_hp);
    } else {
      pair = p.pairs_per_unit - 1 - rank;
    }
  } else {
    it.unit = it.pair_index / p.pairs_per_unit;
    pair = it.pair_index % p.pairs_per_unit;
  }
  it.tile[0] = prefill_tile(p, ms, pair, 0);
  it.tile[1] = prefill_tile(p, ms, pair, 1);
  const KeyRange& a = it.tile[0].kr;
  const KeyRange& b = it.tile[1].kr;
  if (a.t_count == 0 && b.t_count == 0) {
    it.j_first = 0;
    it.j_count = 0;
  } else {
    const int fa = a.t_count ? a.t_first : 0x7fffffff, fb = b.t_count ? b.t_first : 0x7fffffff;
    const int la = a.t_count ? a.t_first + a.t_count - 1 : -1;
    const int lb = b.t_count ? b.t_first + b.t_count - 1 : -1;
    it.j_first = min(fa, fb);
    it.j_count = max(la, lb) - it.j_first + 1;
  }
  if (kSplit && p.splits > 1) {  // this item's share of the key tiles
    // Split s takes [ceil(s J / S), ceil((s + 1) J / S)) of the item's J.
    const int J = it.j_count, S = p.splits;
    const int js = (it.split * J + S - 1) / S, je = ((it.split + 1) * J + S - 1) / S;
    it.j_first += js;
    it.j_count = je - js;
  }
  it.kt0[0] = it.kt0[1] = it.j_first;
  it.kc[0] = it.kc[1] = it.j_count;
  it.busy = it.j_count > 0;
  return it;
}

// The k-th item of this CTA in the persistent loop.  Items sorted heavy
// first (causal / window) go out boustrophedon: round k hands item
// k G + c to CTA c on even rounds and k G + (G - 1 - c) on odd ones, so no
// CTA takes the heaviest item of every round.  The index grows with k.
__device__ __forceinline__ int snake_item(const PrefillParams& p, int k) {
  const int G = (int)gridDim.x, c = (int)blockIdx.x;
  return k * G + ((p.heavy_first && (k & 1)) ? G - 1 - c : c);
}

__device__ __forceinline__ bool tile_active(const PfItem& it, int t, int j) {
  if (it.paired) return j < (t == 0 ? it.kc[0] : it.kc[1]);
  const KeyRange& kr = t == 0 ? it.tile[0].kr : it.tile[1].kr;
  const int jj = it.j_first + j;
  return kr.t_count > 0 && jj >= kr.t_first && jj < kr.t_first + kr.t_count;
}

// Key tile that tile t works on at iteration j.
__device__ __forceinline__ int key_tile(const PfItem& it, int t, int j) {
  return (t == 0 ? it.kt0[0] : it.kt0[1]) + j;
}

// kCapDeg: 0 = no softcap; 5 or 7 = softcap with the row max, with the odd
// polynomial of that degree for tanh of small arguments (5 where the cap is
// small enough for its error, see kTanh5C*); 3 = softcap with the degree-5
// polynomial and a fixed exponent base (PrefillParams::cap_fixed), the only
// softmax path compiled into that kernel.  kSplit: 0 = no key splits (the
// split code is not compiled in); 1 = items cover key-range splits whose
// partials the last CTA of a unit merges (tickets); 2 = paired splits, one
// item per CTA, merged by the unit's thread-block cluster.  Both keep their
// partials in the workspace.  Each kernel holds only its own merge code:
// the ticket merge alone made the clustered kernel slower.
template <int DCH, int kCapDeg, int kSplit>
__global__ void __launch_bounds__(kPfThreads, 1)
    prefill_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v,
                         const __grid_constant__ CUtensorMap tm_o, const PrefillParams p) {
  using C = PrefillCfg<DCH>;
  constexpr bool kCap = kCapDeg != 0;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sq = smem;                   // Q tiles A, B
  uint8_t* ring = smem + C::kQBytes;    // K/V slots
  uint8_t* stage_all = ring + C::kRingBytes;  // output staging, 4 KB per softmax warp
  float2* xchg = (float2*)(stage_all + C::kXchgOffset);
  uint64_t* bars = (uint64_t*)(smem + C::kBarOffset);
  uint64_t* q_full = bars;
  uint64_t* q_empty = bars + 1;
  uint64_t* kv_full = bars + 2;
  uint64_t* kv_empty = kv_full + C::kSlots;
  uint64_t* s_full = kv_empty + C::kSlots;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_done = p_full + 2;  // [t]: every MMA of q tile t in the item has finished
  uint64_t* drain = o_done + 2;
  // Key splits: the four warps of softmax warpgroup t have written their
  // partials (part_done[t]), and the ticket's answer is in merge_flag[t]
  // (flag_ready[t]).
  uint64_t* part_done = drain + 1;
  uint64_t* flag_ready = part_done + 2;
  uint64_t* p_half = flag_ready + 2;  // [t]: P of keys 0..63 of tile t is in TMEM
  uint32_t* tmem_slot = (uint32_t*)(p_half + 2);
  int* merge_flag = (int*)(tmem_slot + 1);  // [2]: 1 merge, 0 not the last, -1 wait gave up

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const MaskSpec ms{p.q_len, p.kv_len, p.causal, p.window};

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < C::kSlots; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 4);  // one arrival per warp of the tile's warpgroup
      mbar_init(&p_half[t], 4);
      mbar_init(&o_done[t], 1);
    }
    mbar_init(drain, 1);
    for (int t = 0; t < 2; ++t) {
      mbar_init(&part_done[t], 128);
      mbar_init(&flag_ready[t], 1);
    }
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
  // P_t (bf16 pairs) overwrites the first 64 columns of S_t.  Named barriers
  // 1 + q (64 threads): warps 4 + q and 8 + q (the same TMEM lane quarter).

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow));
  }
  if (warp == 0 || (kSplit && warp == 2 && p.split_pairs)) {
    // ------------------------------------------------------------ loaders
    // Paired items (split_pairs): K and V have sub-rings of kSlots / 2 slots
    // each, streamed by two threads (warp 0: Q and K, warp 2: V), so a K
    // tile never queues behind a V slot that waits for the softmax.
    // Otherwise warp 0 streams Q and K_j, V_j through the whole ring.
    if (lane == 0) {
      constexpr int kHalf = C::kSlots / 2;
      const bool v_stream = kSplit && warp == 2;
      if (!v_stream) tma_prefetch_map(&tm_q);
      tma_prefetch_map(&tm_k);
      tma_prefetch_map(&tm_v);
      int u = 0;       // K/V tiles issued (ring position, or stream position when paired)
      int nq = 0;      // busy items whose Q was issued
      bool ok = true;
      for (int kk = 0, item = snake_item(p, 0); item < p.n_items && ok;
           ++kk, item = snake_item(p, kk)) {
        const PfItem it = prefill_item<kSplit>(p, ms, item);
        if (!it.busy) continue;
        const int kvh = it.unit % p.kv_heads, bidx = it.unit / p.kv_heads;
        if (!v_stream) {
          // The Q buffer is free once every S of the previous busy item is done.
          if (nq > 0 && !(ok = mbar_wait(q_empty, (nq - 1) & 1, kStatusTimeoutProducer))) break;
          // Paired items share tile 0's Q.
          const int qtiles = it.paired ? 1 : 2;
          int ntiles = 0;
          for (int t = 0; t < qtiles; ++t) ntiles += it.tile[t].nrows > 0 ? 1 : 0;
          mbar_arrive_expect_tx(q_full, ntiles * C::kTileBytes);
          for (int t = 0; t < qtiles; ++t)
            if (it.tile[t].nrows > 0)
              for (int c = 0; c < DCH; ++c)
                tma_load_3d(sq + t * C::kTileBytes + c * C::kBoxBytes, &tm_q, q_full, c * 64,
                            it.tile[t].row0, it.unit);
          ++nq;
        }
        if (it.paired) {
          // Stream order: (A, 0), (B, 0), (A, 1), ... (tile B may end first).
          const int kv = v_stream ? 1 : 0;
          // At the start every CTA asks for its first tiles at once; V is
          // needed one softmax later than Q and K, so it queues behind them.
          if (v_stream && u == 0 &&
              !(ok = mbar_wait(&kv_full[0], 0, kStatusTimeoutProducer)))
            break;
          const CUtensorMap* map = kv ? &tm_v : &tm_k;
          for (int j = 0; j < it.j_count && ok; ++j)
            for (int t = 0; t < 2; ++t) {
              if (!tile_active(it, t, j)) continue;
              const int s = kv * kHalf + u % kHalf;
              if (u >= kHalf &&
                  !(ok = mbar_wait(&kv_empty[s], ((u / kHalf) - 1) & 1, kStatusTimeoutProducer)))
                break;
              uint8_t* dst = ring + s * C::kTileBytes;
              mbar_arrive_expect_tx(&kv_full[s], C::kTileBytes);
              for (int c = 0; c < DCH; ++c)
                tma_load_4d(dst + c * C::kBoxBytes, map, &kv_full[s], c * 64,
                            key_tile(it, t, j) * kPfN, kvh, bidx);
              ++u;
            }
          continue;
        }
        for (int j = 0; j < it.j_count && ok; ++j) {
          const int key0 = key_tile(it, 0, j) * kPfN;
          for (int kv = 0; kv < 2; ++kv) {
            const int s = u % C::kSlots;
            if (u >= C::kSlots &&
                !(ok = mbar_wait(&kv_empty[s], ((u / C::kSlots) - 1) & 1,
                                 kStatusTimeoutProducer)))
              break;
            uint8_t* dst = ring + s * C::kTileBytes;
            mbar_arrive_expect_tx(&kv_full[s], C::kTileBytes);
            for (int c = 0; c < DCH; ++c)
              tma_load_4d(dst + c * C::kBoxBytes, kv ? &tm_v : &tm_k, &kv_full[s], c * 64,
                          key0, kvh, bidx);
            ++u;
          }
        }
      }
      // Drain: never leave with copies in flight.
      if (!v_stream && nq > 0) mbar_wait(q_full, (nq - 1) & 1, kStatusTimeoutProducer);
      if (kSplit && p.split_pairs) {
        const int kv = v_stream ? 1 : 0;
        for (int v = max(0, u - kHalf); v < u; ++v)
          mbar_wait(&kv_full[kv * kHalf + v % kHalf], (v / kHalf) & 1, kStatusTimeoutProducer);
      } else {
        for (int v = max(0, u - C::kSlots); v < u; ++v)
          mbar_wait(&kv_full[v % C::kSlots], (v / C::kSlots) & 1, kStatusTimeoutProducer);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(kPfM, kPfN, 0);
      const uint32_t idesc_o = idesc_bf16_f32(kPfM, p.d_pad, 1);
      const int ksteps = p.d_pad / 16;
      const uint32_t sq_addr = smem_u32(sq);
      const uint32_t ring_addr = smem_u32(ring);
      int ubase = 0;              // ring position of the current item's K_0
      int nq = 0;                 // busy items started (q_full phases)
      int n_act[2] = {0, 0};      // P tiles consumed per q tile (p_full phases)
      bool ok = true;
      for (int kk = 0, item = snake_item(p, 0); item < p.n_items && ok;
           ++kk, item = snake_item(p, kk)) {
        const PfItem it = prefill_item<kSplit>(p, ms, item);
        if (!it.busy) continue;
        if (!(ok = mbar_wait(q_full, nq & 1, kStatusTimeoutMma))) break;
        ++nq;
        int s_left = 0;  // S products still to issue for this item
        int last_j[2] = {-1, -1};  // last key step of each q tile (o_done[t] follows its P.V)
        for (int t = 0; t < 2; ++t)
          for (int j = 0; j < it.j_count; ++j)
            if (tile_active(it, t, j)) {
              ++s_left;
              last_j[t] = j;
            }
        // A q tile without key steps in this item still completes its o_done.
        auto finish_idle_tiles = [&]() {
          for (int t = 0; t < 2; ++t)
            if (last_j[t] < 0) mma_commit(&o_done[t]);
        };
        auto slot_addr = [&](int idx) {
          return ring_addr + ((ubase + idx) % C::kSlots) * C::kTileBytes;
        };
        auto wait_slot = [&](int idx) {
          const int u = ubase + idx;
          return mbar_wait(&kv_full[u % C::kSlots], (u / C::kSlots) & 1, kStatusTimeoutMma);
        };
        auto release = [&](int idx) { mma_commit(&kv_empty[(ubase + idx) % C::kSlots]); };
        // S: both descriptors are built once; the K-steps (ksteps <= 4 * DCH)
        // advance their address fields by compile-time offsets.
        auto issue_s_at = [&](int t, uint32_t kslot) {
          const uint32_t qt = sq_addr + (it.paired ? 0 : t * C::kTileBytes);
          const uint32_t d_tmem = tmem + t * 128;
          const uint64_t qd = sdesc_sw128(qt, 16, 1024);
          const uint64_t kd = sdesc_sw128(kslot, 16, 1024);
          tc_fence_after();
          mma_bf16_ss(d_tmem, qd, kd, idesc_s, 0u);
#pragma unroll
          for (int ks = 1; ks < 4 * DCH; ++ks) {
            if (ks >= ksteps) break;
            const uint32_t off = (ks >> 2) * C::kBoxBytes + (ks & 3) * 32;
            mma_bf16_ss(d_tmem, sdesc_advance(qd, off), sdesc_advance(kd, off), idesc_s, 1u);
          }
          mma_commit(&s_full[t]);
          if (--s_left == 0) mma_commit(q_empty);  // Q no longer read: it may be reloaded
        };
        // P.V: the V descriptor is built once; the K-steps advance its
        // 14-bit address field by compile-time offsets (sdesc_advance).
        // Half h of P.V: keys 64h .. 64h + 63 (K-steps 4h .. 4h + 3).
        auto issue_pv_half = [&](int t, uint32_t vslot, bool first, int h) {
          const uint32_t p_tmem = tmem + t * 128;
          const uint32_t o_tmem = tmem + 256 + t * 128;
          const uint64_t vd = sdesc_sw128(vslot, C::kBoxBytes, 1024);
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < kPfN / 32; ++k) {
            const int ks = h * (kPfN / 32) + k;
            mma_bf16_ts(o_tmem, p_tmem + ks * 8, sdesc_advance(vd, ks * 2048), idesc_o,
                        (first && ks == 0) ? 0u : 1u);
          }
        };
        // P.V in two halves: the first as soon as the softmax has written
        // P of keys 0..63 (p_half), the second after the whole tile (p_full).
        auto issue_pv_at = [&](int t, uint32_t vslot, bool first, int nph) -> bool {
          if (!mbar_wait(&p_half[t], nph & 1, kStatusTimeoutMma)) return false;
          issue_pv_half(t, vslot, first, 0);
          if (!mbar_wait(&p_full[t], nph & 1, kStatusTimeoutMma)) return false;
          issue_pv_half(t, vslot, false, 1);
          return true;
        };
        bool first_pv[2] = {true, true};
        if (it.paired) {
          // K and V sub-rings of kSlots / 2 slots, each filled in the order
          // (A, 0), (B, 0), (A, 1), ...; every slot is released right after
          // its only reader is issued.
          constexpr int kHalf = C::kSlots / 2;
          auto up = [&](int t, int j) { return ubase + j + min(j, it.kc[1]) + t; };
          auto ps = [&](int kv, int pos) { return kv * kHalf + pos % kHalf; };
          auto pwait = [&](int kv, int pos) {
            return mbar_wait(&kv_full[ps(kv, pos)], (pos / kHalf) & 1, kStatusTimeoutMma);
          };
          auto paddr = [&](int kv, int pos) { return ring_addr + ps(kv, pos) * C::kTileBytes; };
          auto prelease = [&](int kv, int pos) { mma_commit(&kv_empty[ps(kv, pos)]); };
          if (!(ok = pwait(0, up(0, 0)))) break;
          issue_s_at(0, paddr(0, up(0, 0)));
          prelease(0, up(0, 0));
          if (tile_active(it, 1, 0)) {
            if (!(ok = pwait(0, up(1, 0)))) break;
            issue_s_at(1, paddr(0, up(1, 0)));
            prelease(0, up(1, 0));
          }
          for (int j = 0; j < it.j_count && ok; ++j) {
            for (int t = 0; t < 2 && ok; ++t) {
              if (!tile_active(it, t, j)) continue;
              if (!(ok = pwait(1, up(t, j)))) break;  // V_t(j)
              if (!(ok = issue_pv_at(t, paddr(1, up(t, j)), first_pv[t], n_act[t]))) break;
              first_pv[t] = false;
              ++n_act[t];
              if (j == last_j[t]) mma_commit(&o_done[t]);
              prelease(1, up(t, j));
              if (tile_active(it, t, j + 1)) {
                if (!(ok = pwait(0, up(t, j + 1)))) break;
                issue_s_at(t, paddr(0, up(t, j + 1)));
                prelease(0, up(t, j + 1));
              }
            }
          }
          if (!ok) break;
          finish_idle_tiles();
          ubase += it.kc[0] + it.kc[1];
          continue;
        }
        auto issue_s = [&](int t, int j) { issue_s_at(t, slot_addr(2 * j)); };
        auto issue_pv = [&](int t, int j, bool first) {
          return issue_pv_at(t, slot_addr(2 * j + 1), first, n_act[t]);
        };

        // Prologue: S(0) of both tiles (K_0's only readers, so its slot is
        // released at once).
        if (!(ok = wait_slot(0))) break;
        if (tile_active(it, 0, 0)) issue_s(0, 0);
        if (tile_active(it, 1, 0)) issue_s(1, 0);
        release(0);
        for (int j = 0; j < it.j_count && ok; ++j) {
          if (!(ok = wait_slot(2 * j + 1))) break;  // V_j
          bool k_next_ready = j + 1 >= it.j_count;
          for (int t = 0; t < 2 && ok; ++t) {
            if (tile_active(it, t, j)) {
              if (!(ok = issue_pv(t, j, first_pv[t]))) break;
              first_pv[t] = false;
              ++n_act[t];
              if (j == last_j[t]) mma_commit(&o_done[t]);
            }
            if (j + 1 < it.j_count && tile_active(it, t, j + 1)) {
              if (!k_next_ready) {
                if (!(ok = wait_slot(2 * (j + 1)))) break;  // K_{j+1}
                k_next_ready = true;
              }
              issue_s(t, j + 1);
            }
          }
          // K_{j+1} must have landed before it can be released.
          if (ok && !k_next_ready) ok = wait_slot(2 * (j + 1));
          if (!ok) break;
          // Release each slot once its last reader is issued: V_j after P.V
          // of iteration j, K_{j+1} after S of j+1.
          release(2 * j + 1);
          if (j + 1 < it.j_count) release(2 * (j + 1));
        }
        if (!ok) break;
        finish_idle_tiles();
        ubase += 2 * it.j_count;
      }
      // Drain: every MMA finished before TMEM can be released.
      mma_commit(drain);
      mbar_wait(drain, 0, kStatusTimeoutMma);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax / epilogue
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsHigh));
    // Warpgroup t (warps 4-7: tile A, 8-11: tile B); thread = row r of its
    // q tile, which is TMEM lane r (warp w reads lane quarter w % 4).
    const int t = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const uint32_t s_tm = tmem + lane_base + t * 128;
    const uint32_t o_tm = tmem + lane_base + 256 + t * 128;
    uint8_t* stage = stage_all + (warp - 4) * 4096;
    // O columns of this thread's row of tile u, col .. col + 15 (warp-collective).
    auto load_o = [&](int u, int col, float (&v)[16]) {
      uint32_t ov[16];
      tmem_ld16(tmem + lane_base + 256 + u * 128 + col, ov);
      tmem_ld_wait();
#pragma unroll
      for (int e = 0; e < 16; ++e) v[e] = __uint_as_float(ov[e]);
    };
    int n_s = 0;      // S tiles consumed (s_full[t] phases)
    int n_busy = 0;   // busy items finished (o_done phases)
    int n_merge = 0;  // split tickets taken by this warpgroup (part_done[t] phases)
    bool ok = true;
    for (int kk = 0, item = snake_item(p, 0); item < p.n_items && ok;
         ++kk, item = snake_item(p, kk)) {
      const PfItem it = prefill_item<kSplit>(p, ms, item);
      const TileInfo ti = t ? it.tile[1] : it.tile[0];
      int lo = 0, hi = -1;  // visible keys of this row (hi < lo: none)
      if (r < ti.nrows) {
        const long long grow = (long long)ti.row0 + r;  // row within the unit
        const int qpos = p.kv_len - p.q_len + (int)(grow % p.q_len);
        lo = first_key(ms, qpos);
        hi = last_key(ms, qpos);
      }
      float m = -INFINITY;  // running max (log2 domain)
      float l = 0.f;        // running sum
      int act = 0;          // key tiles consumed in this item (the same in the whole warpgroup)
      for (int j = 0; j < it.j_count; ++j) {
        if (!tile_active(it, t, j)) continue;
        const int ktile0 = key_tile(it, t, j) * kPfN;
        const bool need_mask = !(ktile0 >= ti.kr.all_lo && ktile0 + kPfN - 1 <= ti.kr.all_hi);
        ok = __all_sync(0xffffffffu, mbar_wait(&s_full[t], n_s & 1, kStatusTimeoutSoftmax));
        ++n_s;
        if (!ok) break;
        tc_fence_after();
        // Visible columns of this row: c is hidden iff (unsigned)(c - vlo) >
        // vspan (the range clamped to the tile; an empty range hides all).
        const int clo = max(lo - ktile0, 0), chi = min(hi - ktile0, kPfN - 1);
        const int vlo = chi >= clo ? clo : kPfN;
        const unsigned vspan = chi >= clo ? (unsigned)(chi - clo) : 0u;
        // Pass 1, 32 scores at a time: the row's max over its visible keys
        // and, with a softcap, the raw scores' range (when every |x / s| of
        // the warp's rows is <= 1/2, tanh runs as an odd polynomial on the
        // FMA pipe).  On tiles with a mask the hidden scores become -inf and
        // are written back, so pass 2 is the same code on every tile.
        if constexpr (kCapDeg == 3) {
          {
            // One pass over the scores, no row max: y = cap(x) - cap_base.
            // Per 32-key group, the warp takes the degree-5 polynomial when
            // every |x * cap_in| <= 1/2 (hidden keys as -inf then give p = 0),
            // else the hardware tanh with hidden keys zeroed by column.
            const float base = p.cap_base;
            m = base;
            const f2 nb = f2_pack(-base, -base);
            const float ci2 = p.cap_in * p.cap_in, cc = p.cap_out * p.cap_in;
            const f2 q0 = f2_pack(cc * kTanh5C1, cc * kTanh5C1);
            const f2 q1 = f2_pack(cc * ci2 * kTanh5C3, cc * ci2 * kTanh5C3);
            const f2 q2 = f2_pack(cc * ci2 * ci2 * kTanh5C5, cc * ci2 * ci2 * kTanh5C5);
            f2 acc[4] = {0ull, 0ull, 0ull, 0ull};
            auto group = [&](uint32_t(&sv)[32], int g) {
              float am = fmaxf(fabsf(__uint_as_float(sv[0])), fabsf(__uint_as_float(sv[1])));
#pragma unroll
              for (int c = 2; c < 32; c += 2)
                am = fmax3(am, fabsf(__uint_as_float(sv[c])), fabsf(__uint_as_float(sv[c + 1])));
              const bool poly = __all_sync(0xffffffffu, am * p.cap_in <= 0.5f);
              if (need_mask) {
#pragma unroll
                for (int c = 0; c < 32; ++c)
                  if ((unsigned)(32 * g + c - vlo) > vspan) sv[c] = __float_as_uint(-INFINITY);
              }
              uint32_t pk[16];
              if (poly) {
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                  const f2 v = f2_pack(__uint_as_float(sv[2 * c]), __uint_as_float(sv[2 * c + 1]));
                  const f2 v2 = f2_mul(v, v);
                  const f2 pv = exp2_mufu_x2(f2_fma(v, f2_fma(f2_fma(q2, v2, q1), v2, q0), nb));
                  acc[c & 3] = f2_add(acc[c & 3], pv);
                  pk[c] = pack_bf16_f2(pv);
                }
              } else {
                const float co = p.cap_out, ci = p.cap_in;
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                  const float a = __uint_as_float(sv[2 * c]), b = __uint_as_float(sv[2 * c + 1]);
                  f2 pv = exp2_mufu_x2(f2_pack(fmaf(co, tanh_fast(a * ci), -base),
                                               fmaf(co, tanh_fast(b * ci), -base)));
                  if (need_mask) {
                    float pa, pb;
                    f2_unpack(pv, pa, pb);
                    const int col = 32 * g + 2 * c;
                    pv = f2_pack((unsigned)(col - vlo) > vspan ? 0.f : pa,
                                 (unsigned)(col + 1 - vlo) > vspan ? 0.f : pb);
                  }
                  acc[c & 3] = f2_add(acc[c & 3], pv);
                  pk[c] = pack_bf16_f2(pv);
                }
              }
              tmem_st16(s_tm + 16 * g, pk);
            };
            uint32_t b0[32], b1[32];
            tmem_ld32(s_tm, b0);
            tmem_ld_wait();
#pragma unroll 1
            for (int g = 0; g < 4; g += 2) {
              tmem_ld32(s_tm + 32 * (g + 1), b1);
              group(b0, g);
              tmem_ld_wait();
              if (g + 2 < 4) tmem_ld32(s_tm + 32 * (g + 2), b0);
              group(b1, g + 1);
              if (g + 2 < 4) tmem_ld_wait();
              if (g == 0) {  // P of keys 0..63 written: the first half of P.V may start
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_half[t]);
              }
            }
            float a0, a1, c0, c1, d0, d1, e0, e1;
            f2_unpack(acc[0], a0, a1);
            f2_unpack(acc[1], c0, c1);
            f2_unpack(acc[2], d0, d1);
            f2_unpack(acc[3], e0, e1);
            l += ((a0 + a1) + (c0 + c1)) + ((d0 + d1) + (e0 + e1));
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[t]);
            ++act;
            continue;
          }
        }
        bool small_y = false;
        float mraw = -INFINITY;
        {
          float amax = 0.f;  // max |x| over the raw scores (softcap check)
#pragma unroll 1
          for (int g = 0; g < 4; ++g) {
            uint32_t sr[32];
            tmem_ld32(s_tm + 32 * g, sr);
            tmem_ld_wait();
            if constexpr (kCap) {
#pragma unroll
              for (int c = 0; c < 32; c += 2)
                amax = fmax3(amax, fabsf(__uint_as_float(sr[c])), fabsf(__uint_as_float(sr[c + 1])));
            }
            if (need_mask) {
#pragma unroll
              for (int c = 0; c < 32; ++c)
                if ((unsigned)(32 * g + c - vlo) > vspan) sr[c] = __float_as_uint(-INFINITY);
              tmem_st32(s_tm + 32 * g, sr);
            }
            float m2[2] = {fmaxf(__uint_as_float(sr[0]), __uint_as_float(sr[1])),
                           fmaxf(__uint_as_float(sr[2]), __uint_as_float(sr[3]))};
#pragma unroll
            for (int c = 4; c < 32; c += 4) {
              m2[0] = fmax3(m2[0], __uint_as_float(sr[c]), __uint_as_float(sr[c + 1]));
              m2[1] = fmax3(m2[1], __uint_as_float(sr[c + 2]), __uint_as_float(sr[c + 3]));
            }
            mraw = fmax3(mraw, m2[0], m2[1]);
          }
          if (need_mask) tmem_st_wait();  // pass 2 reads the masked scores
          if constexpr (kCap) small_y = __all_sync(0xffffffffu, amax * p.cap_in <= 0.5f);
        }
        const float mt = mraw == -INFINITY ? -INFINITY
                         : kCap ? p.cap_out * tanh_fast(mraw * p.cap_in)
                                : mraw * p.logit_scale;
        // Rescale only when the max grew by more than 2^8 (or was -inf): the
        // stale max keeps p <= 256, and O / l stays consistent.
        const float m_new = fmaxf(m, mt);
        const bool need =
            (m_new > m + kRescaleThreshold) || (m == -INFINITY && m_new != -INFINITY);
        const float alpha = need ? ex2(m - m_new) : 1.0f;  // 0 when m = -inf
        if (need) {
          l *= alpha;
          m = m_new;
        }
        if (__any_sync(0xffffffffu, need) && act > 0) {
          // This row of O_t (tcgen05.ld / st are warp-collective).
          for (int c0 = 0; c0 < p.d_pad; c0 += 16) {
            uint32_t ov[16];
            tmem_ld16(o_tm + c0, ov);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 16; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
            tmem_st16(o_tm + c0, ov);
          }
          tmem_st_wait();
        }
        const float base = m == -INFINITY ? 0.f : m;
        // Pass 2: p = 2^(logit - base) as bf16 pairs into TMEM over S, 32
        // keys at a time (two groups per turn of a loop; the next group's
        // read is in flight while one is computed): P of keys 32g .. 32g + 31
        // lands in columns [16g, 16g + 16), whose scores were read before.
        // Pairs [kEmuFrom, 16) of each group take the FMA-pipe 2^x.  A
        // hidden key's score is -inf and gives p = 0; the logit transforms
        // that do not carry -inf through (`explicit_hidden`) zero it by
        // column range instead.
        f2 acc[4] = {0ull, 0ull, 0ull, 0ull};
        auto emit = [&](auto logit2, auto explicit_hidden) {
          constexpr bool kHid = decltype(explicit_hidden)::value;
          auto group = [&](const uint32_t(&sv)[32], int g) {
            uint32_t pk[16];
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const f2 y = logit2(f2_pack(__uint_as_float(sv[2 * c]), __uint_as_float(sv[2 * c + 1])));
              f2 pv = (!kCap && c >= kEmuFrom) ? exp2_poly_x2(y) : exp2_mufu_x2(y);
              if constexpr (kHid) {
                float a, b;
                f2_unpack(pv, a, b);
                const int col = 32 * g + 2 * c;
                pv = f2_pack((unsigned)(col - vlo) > vspan ? 0.f : a,
                             (unsigned)(col + 1 - vlo) > vspan ? 0.f : b);
              }
              acc[c & 3] = f2_add(acc[c & 3], pv);
              pk[c] = pack_bf16_f2(pv);
            }
            tmem_st16(s_tm + 16 * g, pk);
          };
          uint32_t b0[32], b1[32];
          tmem_ld32(s_tm, b0);
          tmem_ld_wait();
#pragma unroll 1
          for (int g = 0; g < 4; g += 2) {
            tmem_ld32(s_tm + 32 * (g + 1), b1);
            group(b0, g);
            tmem_ld_wait();
            if (g + 2 < 4) tmem_ld32(s_tm + 32 * (g + 2), b0);
            group(b1, g + 1);
            if (g + 2 < 4) tmem_ld_wait();
            if (g == 0) {  // P of keys 0..63 written: the first half of P.V may start
              tmem_st_wait();
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&p_half[t]);
            }
          }
        };
        using Yes = std::true_type;
        using No = std::false_type;
        const f2 nb = f2_pack(-base, -base);
        if constexpr (!kCap) {
          const f2 sc = f2_pack(p.logit_scale, p.logit_scale);
          emit([&](f2 v) { return f2_fma(v, sc, nb); }, No());
        } else if (small_y) {
          // cap_out * tanh(x * cap_in) = x * Q(x^2), the odd polynomial with
          // cap_in^(2k+1) * cap_out folded into its coefficients.  Degree 5:
          // its top coefficient is positive, so x = -inf gives -inf.
          const float ci2 = p.cap_in * p.cap_in, cc = p.cap_out * p.cap_in;
          if constexpr (kCapDeg == 5) {
            const f2 q0 = f2_pack(cc * kTanh5C1, cc * kTanh5C1);
            const f2 q1 = f2_pack(cc * ci2 * kTanh5C3, cc * ci2 * kTanh5C3);
            const f2 q2 = f2_pack(cc * ci2 * ci2 * kTanh5C5, cc * ci2 * ci2 * kTanh5C5);
            emit([&](f2 v) {
              const f2 v2 = f2_mul(v, v);
              return f2_fma(v, f2_fma(f2_fma(q2, v2, q1), v2, q0), nb);
            }, No());
          } else {
            const f2 q0 = f2_pack(cc * kTanhC1, cc * kTanhC1);
            const f2 q1 = f2_pack(cc * ci2 * kTanhC3, cc * ci2 * kTanhC3);
            const f2 q2 = f2_pack(cc * ci2 * ci2 * kTanhC5, cc * ci2 * ci2 * kTanhC5);
            const f2 q3 = f2_pack(cc * ci2 * ci2 * ci2 * kTanhC7, cc * ci2 * ci2 * ci2 * kTanhC7);
            emit([&](f2 v) {
              const f2 v2 = f2_mul(v, v);
              return f2_fma(v, f2_fma(f2_fma(f2_fma(q3, v2, q2), v2, q1), v2, q0), nb);
            }, Yes());
          }
        } else {
          // Large arguments (rare): the hardware tanh, which maps -inf to -1.
          const float co = p.cap_out, ci = p.cap_in;
          emit([&](f2 v) {
            float a, b;
            f2_unpack(v, a, b);
            return f2_pack(fmaf(co, tanh_fast(a * ci), -base), fmaf(co, tanh_fast(b * ci), -base));
          }, Yes());
        }
        {
          float a0, a1, b0, b1, c0, c1, d0, d1;
          f2_unpack(acc[0], a0, a1);
          f2_unpack(acc[1], b0, b1);
          f2_unpack(acc[2], c0, c1);
          f2_unpack(acc[3], d0, d1);
          l += ((a0 + a1) + (b0 + b1)) + ((c0 + c1) + (d0 + d1));
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[t]);
        ++act;
      }
      // Paired items (every item of a launch, or none): the two warpgroups
      // meet at a named barrier below, so a warpgroup that gave up on a wait
      // still goes there (with ok = false) instead of leaving at once.
      // Fixed-base softcap: a row without a visible key keeps m = -inf.
      if constexpr (kCapDeg == 3)
        if (!(l > 0.f)) m = -INFINITY;
      const bool pair_x = kSplit && it.paired;
      if (!ok && !pair_x) break;
      // ---- epilogue.  The next item's first P.V of this tile may overwrite
      // O only after this warpgroup's next P arrival, which follows these
      // (waited) TMEM loads in program order.
      if (it.busy) {
        const uint32_t ph = n_busy & 1;
        ++n_busy;
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&o_done[t], ph, kStatusTimeoutEpilogue));
        // Paired items: this warpgroup also reads the other tile's O.
        if (ok && pair_x)
          ok = __all_sync(0xffffffffu, mbar_wait(&o_done[1 - t], ph, kStatusTimeoutEpilogue));
        if (!ok && !pair_x) break;
      }
      tc_fence_after();
      // Write this warp's 32 rows, columns [c0, c0 + 64), as bf16 through its
      // 128B-swizzled 32-row staging box and one TMA store (rows past the
      // unit's end are not written).  value16(col, v) fills v with the fp32
      // outputs of columns col .. col + 15.
      auto store_box = [&](const TileInfo& tile, int c0, auto value16) {
        if (lane == 0) bulk_wait_read();  // the previous store has read the box
        __syncwarp();
        const int cw = min(64, p.d_pad - c0);
        for (int c1 = 0; c1 < cw; c1 += 16) {
          float v[16];
          value16(c0 + c1, v);
#pragma unroll
          for (int g = 0; g < 2; ++g) {  // 8 columns = one 16-byte chunk
            const uint4 w = make_uint4(pack_bf16(v[8 * g], v[8 * g + 1]),
                                       pack_bf16(v[8 * g + 2], v[8 * g + 3]),
                                       pack_bf16(v[8 * g + 4], v[8 * g + 5]),
                                       pack_bf16(v[8 * g + 6], v[8 * g + 7]));
            *reinterpret_cast<uint4*>(stage + sw128(lane, (c1 >> 3) + g)) = w;
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_3d(&tm_o, stage, c0, tile.row0 + quarter * 32, it.unit);
          bulk_commit();
        }
      };
      if constexpr (!kSplit) {
        if (ti.nrows > 0 && quarter * 32 < ti.nrows) {
          const bool have = act > 0;  // warp-uniform
          const bool live = have && m != -INFINITY && l > 0.f;
          const float inv = live ? 1.0f / l : 0.f;
          for (int c0 = 0; c0 < p.d_pad; c0 += 64)
            store_box(ti, c0, [&](int col, float (&v)[16]) {
              if (have) {
                load_o(t, col, v);
#pragma unroll
                for (int e = 0; e < 16; ++e) v[e] = live ? v[e] * inv : 0.f;
              } else {
#pragma unroll
                for (int e = 0; e < 16; ++e) v[e] = 0.f;
              }
            });
        }
      } else {
        // ---- key splits.  Each split leaves a partial per row: O
        // (unnormalised, fp32), m and l.  Unpaired items: warpgroup t writes
        // the partial of its own q tile, all columns.  Paired items (tiles A
        // and B are two splits of the same rows): the two warpgroups swap
        // their rows' (m, l), combine both tiles' O into one partial, and
        // each writes columns [64t, 64t + 64) of it.  One ticket per (row
        // tile, warpgroup); in the CTA that brings the last partial, the four
        // warps of the warpgroup merge all of them in partial order
        // (deterministic), sharing the rows and columns between them.
        const bool paired = it.paired;
        float mo = -INFINITY, lo_ = 0.f;  // the other tile's (m, l) (paired)
        if (paired) {
          // Warps 4 + q and 8 + q hold the same rows.  The first barrier
          // keeps this write behind the partner's read of the previous
          // item's value; the second publishes it and ANDs the two ok flags.
          tc_fence_before();
          named_bar_sync(1 + quarter, 64);
          xchg[t * kPfM + r] = make_float2(m, l);
          ok = named_bar_and(1 + quarter, 64, ok);
          tc_fence_after();
          const float2 other = xchg[(1 - t) * kPfM + r];
          mo = other.x;
          lo_ = other.y;
          if (!ok) break;
        }
        const TileInfo& rt = it.tile[0];  // the row tile of a paired item
        const TileInfo& wt = paired ? rt : ti;
        const int cw0 = paired ? min(64 * t, p.d_pad) : 0;
        const int cw1 = paired ? min(64 * t + 64, p.d_pad) : p.d_pad;
        const int hh = paired ? t : 0;  // (m, l) and ticket slot
        const int np = paired ? p.splits / 2 : p.splits;
        const int psplit = paired ? it.split / 2 : it.split;
        if (wt.nrows > 0) {  // the same for every warp of the warpgroup
          const int ptile = paired ? it.pair_index : it.pair_index * 2 + t;
          const long long blk = (long long)ptile * np;
          auto po_of = [&](int sp) {
            return reinterpret_cast<float4*>(p.ws_o + (blk + sp) * (long long)p.d_pad * kPfM);
          };
          auto ml_of = [&](int sp) { return p.ws_ml + ((blk + sp) * 2 + hh) * 2 * kPfM; };
          if (quarter * 32 < wt.nrows && cw0 < cw1) {
            // Tile A = this warpgroup's (paired: t = 0) or the only tile.
            const int act_a = paired ? it.kc[0] : act, act_b = paired ? it.kc[1] : 0;
            const float ma = paired ? (t ? mo : m) : m, la = paired ? (t ? lo_ : l) : l;
            const float mb = paired ? (t ? m : mo) : -INFINITY, lb = paired ? (t ? l : lo_) : 0.f;
            const bool ha = act_a > 0 && ma != -INFINITY;
            const bool hb = act_b > 0 && mb != -INFINITY;
            float mc = ha ? ma : -INFINITY;
            if (hb) mc = fmaxf(mc, mb);
            const float wa = ha ? ex2(ma - mc) : 0.f;
            const float wb = hb ? ex2(mb - mc) : 0.f;
            const float L = wa * la + (hb ? wb * lb : 0.f);
            const int ua = paired ? 0 : t;  // TMEM O of tile A
            float4* po = po_of(psplit);
            for (int c0 = cw0; c0 < cw1; c0 += 16) {
              float v[16];
#pragma unroll
              for (int e = 0; e < 16; ++e) v[e] = 0.f;
              if (act_a > 0) {  // warp-uniform
                float a[16];
                load_o(ua, c0, a);
#pragma unroll
                for (int e = 0; e < 16; ++e) v[e] = wa * a[e];
              }
              if (act_b > 0) {
                float b[16];
                load_o(1, c0, b);
#pragma unroll
                for (int e = 0; e < 16; ++e) v[e] = fmaf(wb, b[e], v[e]);
              }
#pragma unroll
              for (int g = 0; g < 4; ++g) {
                const float4 f = make_float4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
                po[(c0 / 4 + g) * kPfM + r] = f;
              }
            }
            float* pml = ml_of(psplit);
            pml[r] = ha || hb ? mc : -INFINITY;
            pml[kPfM + r] = L;
          }
          if constexpr (kSplit == 1) {
            // The ticket: every thread's partial is visible device-wide before
            // one thread of the warpgroup counts it (bounded waits: a warp that
            // gave up elsewhere makes the others give up here, not hang).
            __threadfence();
            mbar_arrive(&part_done[t]);
            const uint32_t mph = n_merge & 1;
            ++n_merge;
            unsigned int* tk = p.tickets + ptile * 2 + hh;
            if (quarter == 0 && lane == 0) {
              int f = -1;
              if (mbar_wait(&part_done[t], mph, kStatusTimeoutEpilogue))
                f = atomicAdd(tk, 1u) == (unsigned)(np - 1) ? 1 : 0;
              merge_flag[t] = f;
              mbar_arrive(&flag_ready[t]);
            }
            const int flag =
                __all_sync(0xffffffffu, mbar_wait(&flag_ready[t], mph, kStatusTimeoutEpilogue))
                    ? *(volatile int*)&merge_flag[t]
                    : -1;
            if (flag < 0) {
              ok = false;
              break;
            }
            if (flag == 1) {
              __threadfence();
              if (quarter == 0 && lane == 0) atomicExch(tk, 0u);  // ready for the next call
              // Work of this warp: row group rg (32 rows), column part `part`
              // of [cw0, cw1) (whole 16-column chunks).  Fewer than three row
              // groups: the idle warps take column parts instead.
              const int nq = (wt.nrows + 31) / 32;
              const int parts = nq == 1 ? 4 : nq == 2 ? 2 : 1;
              const int rg = parts == 1 ? quarter : quarter % nq;
              const int part = parts == 1 ? 0 : quarter / nq;
              const int nch = (cw1 - cw0) / 16;
              const int cb = cw0 + 16 * (nch * part / parts);
              const int ce = cw0 + 16 * (nch * (part + 1) / parts);
              if (rg < nq && cb < ce) {
                const int row = rg * 32 + lane;  // < 128: partial rows past nrows exist
                // Row max and row sum over the partials in one pass, eight
                // (m, l) loads in flight at a time; the sum is rescaled when a
                // later batch raises the max.
                float M = -INFINITY, Ls = 0.f;
                for (int sp0 = 0; sp0 < np; sp0 += 8) {
                  float mv[8], lv[8];
#pragma unroll
                  for (int i = 0; i < 8; ++i) {
                    const bool in = sp0 + i < np;
                    mv[i] = in ? __ldcg(ml_of(sp0 + i) + row) : -INFINITY;
                    lv[i] = in ? __ldcg(ml_of(sp0 + i) + kPfM + row) : 0.f;
                  }
                  float mb8 = M;
#pragma unroll
                  for (int i = 0; i < 8; ++i) mb8 = fmaxf(mb8, mv[i]);
                  if (mb8 != -INFINITY) {
                    if (M != -INFINITY) Ls *= ex2(M - mb8);
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                      Ls += mv[i] == -INFINITY ? 0.f : ex2(mv[i] - mb8) * lv[i];
                    M = mb8;
                  }
                }
                const float inv = Ls > 0.f ? 1.0f / Ls : 0.f;
                __nv_bfloat16* orow =
                    p.o + ((long long)it.unit * p.rows + wt.row0 + row) * p.head_dim;
                for (int col = cb; col < ce; col += 16) {
                  float v[16];
#pragma unroll
                  for (int e = 0; e < 16; ++e) v[e] = 0.f;
                  // Eight partials per batch: their m and O loads all in
                  // flight together (past the last partial the loads read
                  // partial 0 with weight 0).
                  for (int sp0 = 0; sp0 < np; sp0 += 8) {
                    float mv[8];
                    float x8[8][16];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                      const int sp = sp0 + i < np ? sp0 + i : 0;
                      mv[i] = sp0 + i < np ? __ldcg(ml_of(sp) + row) : -INFINITY;
                      const float4* src = po_of(sp) + row;
#pragma unroll
                      for (int g = 0; g < 4; ++g) {
                        const float4 f = __ldcg(src + (col / 4 + g) * kPfM);
                        x8[i][4 * g] = f.x;
                        x8[i][4 * g + 1] = f.y;
                        x8[i][4 * g + 2] = f.z;
                        x8[i][4 * g + 3] = f.w;
                      }
                    }
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                      const float w = mv[i] == -INFINITY ? 0.f : ex2(mv[i] - M) * inv;
#pragma unroll
                      for (int e = 0; e < 16; ++e) v[e] = fmaf(w, x8[i][e], v[e]);
                    }
                  }
                  if (row < wt.nrows) {
                    // 8 columns (16 bytes) at a time; head_dim is a multiple of 8.
#pragma unroll
                    for (int g = 0; g < 2; ++g)
                      if (col + 8 * g < p.head_dim)
                        *reinterpret_cast<uint4*>(orow + col + 8 * g) = make_uint4(
                            pack_bf16(v[8 * g], v[8 * g + 1]), pack_bf16(v[8 * g + 2], v[8 * g + 3]),
                            pack_bf16(v[8 * g + 4], v[8 * g + 5]),
                            pack_bf16(v[8 * g + 6], v[8 * g + 7]));
                  }
                }
              }
            }
          }
        }
      }
    }
    if (lane == 0) bulk_wait_all();  // stores done before the CTA exits
  }

  // ---------------------------------------------------------------- cluster merge
  // Every thread of every CTA reaches the cluster barrier (no role leaves the
  // kernel early; all waits above are bounded).  Its release / acquire makes
  // every CTA's partial in the workspace visible to the cluster; then the
  // softmax warps of CTA `rank` merge column groups [g0, g1) of every row
  // from the partials of all CTAs of the cluster, in rank order, reading
  // them from L2.
  if constexpr (kSplit) {
    if constexpr (kSplit == 2) {
      __syncwarp();
      cluster_sync();
      if (warp >= 4) {
        const int csize = p.cluster_merge;
        const uint32_t rank = cluster_ctarank();
        const int G = p.d_pad / 4;
        const int g0 = (int)rank * G / csize, g1 = ((int)rank + 1) * G / csize, ng = g1 - g0;
        const int nrows = min(kPfM, p.rows);
        const int unit = (int)blockIdx.x / csize;
        const long long blk = (long long)unit * csize;  // the unit's partial slots
        // Consecutive threads take consecutive rows: coalesced partial loads.
        for (int i = threadIdx.x - 128; i < nrows * ng; i += 256) {
          const int row = i % nrows, g = g0 + i / nrows;
          float mv[8], lv[8];
          float4 f[8];
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            mv[c] = -INFINITY;
            lv[c] = 0.f;
            f[c] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (c < csize) {
              const float* ml = p.ws_ml + (blk + c) * 2 * 2 * kPfM;
              mv[c] = __ldcg(ml + row);
              lv[c] = __ldcg(ml + kPfM + row);
              f[c] = __ldcg(reinterpret_cast<const float4*>(p.ws_o + (blk + c) * (long long)p.d_pad * kPfM) +
                            g * kPfM + row);
            }
          }
          float M = -INFINITY;
#pragma unroll
          for (int c = 0; c < 8; ++c) M = fmaxf(M, mv[c]);
          float Ls = 0.f;
          float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const float w = mv[c] == -INFINITY ? 0.f : ex2(mv[c] - M);
            Ls = fmaf(w, lv[c], Ls);
            acc.x = fmaf(w, f[c].x, acc.x);
            acc.y = fmaf(w, f[c].y, acc.y);
            acc.z = fmaf(w, f[c].z, acc.z);
            acc.w = fmaf(w, f[c].w, acc.w);
          }
          const float inv = Ls > 0.f ? 1.0f / Ls : 0.f;
          if (4 * g < p.head_dim) {  // head_dim is a multiple of 8
            __nv_bfloat16* dst = p.o + ((long long)unit * p.rows + row) * p.head_dim + 4 * g;
            *reinterpret_cast<uint2*>(dst) =
                make_uint2(pack_bf16(acc.x * inv, acc.y * inv), pack_bf16(acc.z * inv, acc.w * inv));
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
