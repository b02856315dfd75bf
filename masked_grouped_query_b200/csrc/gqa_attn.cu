// gqa_attn.cu -- host side of libgqa_attn.so: argument validation, planning,
// tensor maps, workspace and launches behind the C ABI of gqa_attn.h.
//
// Single translation unit: the kernels are included below.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>
#include <vector>

#include "gqa_attn.h"
#include "status.cuh"
#include "ptx.cuh"
#include "mask.cuh"
#include "decode_splitkv.cuh"
#include "prefill_sm100.cuh"
#include "kv_append.cuh"
#include "selftest.cuh"

namespace {

using namespace gqa;

constexpr float kLog2e = 1.4426950408889634f;

// ------------------------------------------------------------------ device
struct DeviceInfo {
  bool probed = false;
  int sms = 0, major = 0, minor = 0;
  int smem_optin = 0;
  bool decode_attr[10] = {};  // per instantiation: [0, 8) 3/2-stage, [8, 10) 5-stage
  bool prefill_attr[24] = {};  // per (DCH, softcap code, split mode) instantiation
  int append_blocks[4] = {};    // resident kv_append blocks per SM, per instantiation
  bool append_runs_ready[4] = {};  // staged-runs kernel's smem attribute set
  // Clusters of n CTAs of a split instantiation that can be resident at once
  // (cudaOccupancyMaxActiveClusters); -1 = not asked yet.
  int cluster_max[24][9];
  DeviceInfo() {
    for (auto& a : cluster_max)
      for (int& n : a) n = -1;
  }
};

std::mutex g_mu;
DeviceInfo g_dev[64];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::atomic<int> g_force_path{0};
std::atomic<int> g_no_cluster{0};
std::atomic<int> g_force_tps{0};
std::atomic<int> g_force_pf_splits{0};
std::atomic<int> g_force_two_pass{0};  // 1: softcap kernels always take the row max first

int device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return GQA_ATTN_ERR_DEVICE;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.probed) {
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
            cudaSuccess)
      return GQA_ATTN_ERR_DEVICE;
    d.probed = true;
  }
  if (d.major != 10) return GQA_ATTN_ERR_DEVICE;
  if (!g_encode) {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
      return GQA_ATTN_ERR_DEVICE;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  *out = &d;
  return GQA_ATTN_OK;
}

// ------------------------------------------------------------------ problem
struct Problem {
  int batch, q_len, kv_len, hq, hkv, d, causal, window;
  float softcap;
  int group;
  long long units;  // batch * hkv
  long long rows;   // group * q_len  (rows per unit)
  long long kv_alloc;  // key slots allocated per (batch, kv head): kv_len, or a cache's slots
  int kv_seq_major;    // 0: k/v [batch][hkv][kv_alloc][d]; 1: [batch][kv_alloc][hkv][d]
  int ring;            // ring of `ring` slots (key j in slot j % ring); 0: keys in order
  // KV-cache append fused into the split-KV decode kernel (app_count > 0).
  int app_count = 0, app_pos = 0, app_new_f32 = 0, app_new_head_major = 0;
  const void* app_new_k = nullptr;
  const void* app_new_v = nullptr;
};

int validate(int batch, int q_len, int kv_len, int hq, int hkv, int d, int causal, int window,
             float softcap, Problem* pr) {
  if (batch < 0 || q_len < 0 || kv_len < 0 || hq < 1 || hkv < 1) return GQA_ATTN_ERR_BAD_SHAPE;
  if (hq % hkv != 0) return GQA_ATTN_ERR_HEAD_RATIO;
  if (d < 8 || d > 256 || d % 8 != 0) return GQA_ATTN_ERR_HEAD_DIM;
  if (!(softcap >= 0.0f) || std::isinf(softcap)) return GQA_ATTN_ERR_SOFTCAP;
  pr->batch = batch;
  pr->q_len = q_len;
  pr->kv_len = kv_len;
  pr->hq = hq;
  pr->hkv = hkv;
  pr->d = d;
  pr->causal = causal ? 1 : 0;
  pr->window = window > 0 ? window : 0;
  pr->softcap = softcap;
  pr->group = hq / hkv;
  pr->units = (long long)batch * hkv;
  pr->rows = (long long)pr->group * q_len;
  pr->kv_alloc = kv_len;
  pr->kv_seq_major = 0;
  pr->ring = 0;
  // Index limits: element offsets are 64-bit, rows per unit and TMA
  // coordinates are 32-bit, the flattened grid is < 2^31.
  const long long q_elems = (long long)batch * hq * (long long)q_len * d;
  const long long kv_elems = (long long)batch * hkv * (long long)kv_len * d;
  if (pr->rows > 0x7fffffffLL || pr->units > 0x7fffffffLL || q_elems < 0 || kv_elems < 0 ||
      (long long)batch * hq > (1LL << 40) || q_elems > (1LL << 56) || kv_elems > (1LL << 56))
    return GQA_ATTN_ERR_TOO_LARGE;
  return GQA_ATTN_OK;
}

// ------------------------------------------------------------------ plan
enum Path { kPathNone = 0, kPathDecode = 1, kPathPrefill = 2, kPathZero = 3 };

struct Plan {
  int path = kPathNone;
  int splits = 1, tps = 1;
  int row_blocks = 0, block_rows = 0;
  int ks = 8;
  int max_tiles = 0;
  long long ctas = 0;
  int dch = 2, d_pad = 128;           // prefill: TMA boxes per tile, padded head_dim
  int tiles_per_unit = 0, pairs_per_unit = 0, pair_heads = 0, split_pairs = 0;
  size_t ws_bytes = 0;      // split partials (o_s, lse_s)
  size_t off_lse = 0;
  size_t ticket_bytes = 0;  // split tickets (kept zero between calls)
};

thread_local char g_detail[160] = "";

// Remember which CUDA call failed (readable with gqa_attn_last_error_detail).
int cuda_fail(const char* where, cudaError_t e, int code) {
  snprintf(g_detail, sizeof g_detail, "%s: %s (%s)", where, cudaGetErrorName(e),
           cudaGetErrorString(e));
  return code;
}

inline long long ceil_div(long long a, long long b) { return (a + b - 1) / b; }
inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Longest key split of the small-row-block decode plan, in key tiles.
constexpr int kDecMaxSplitTiles = 128;

int plan_decode(const Problem& pr, const DeviceInfo& dev, Plan* pl) {
  pl->path = kPathDecode;
  pl->ks = pr.d <= 64 ? 4 : pr.d <= 128 ? 8 : pr.d <= 192 ? 12 : 16;
  pl->row_blocks = (int)ceil_div(pr.rows, kDecRows);
  pl->block_rows = (int)(pr.rows < kDecRows ? pr.rows : kDecRows);
  const MaskSpec ms{pr.q_len, pr.kv_len, pr.causal, pr.window};
  const int k_base = pr.ring ? ring_k_base(pr.kv_len, pr.ring, kDecTile) : 0;
  int max_tiles = 0;
  for (int rb = 0; rb < pl->row_blocks; ++rb) {
    const long long r0 = (long long)rb * kDecRows;
    const int nr = (int)((pr.rows - r0) < kDecRows ? (pr.rows - r0) : kDecRows);
    const KeyRange kr = key_range_from(ms, r0, nr, kDecTile, k_base);
    if (kr.t_count > max_tiles) max_tiles = kr.t_count;
  }
  pl->max_tiles = max_tiles;
  const long long base = pr.units * pl->row_blocks;
  int tps;
  const int forced = g_force_tps.load();
  if (max_tiles == 0) {
    tps = 1;
  } else if (forced > 0) {
    tps = forced;
  } else {
    // Splits per row block, measured on B200 (L2 flushed).  Small row
    // blocks (keys-as-M variant): about one CTA per SM in total, since every
    // extra split adds partial traffic and a merge at the end, but no split
    // longer than kDecMaxSplitTiles tiles (long caches keep several splits per
    // unit so that the grid still has a second CTA per SM to switch to).
    // Larger row blocks (one CTA per SM, partial traffic of 64 rows per
    // split): about two thirds of a wave.
    const bool small = pl->block_rows <= 8;
    const double per_sm = small ? 1.0 : 0.65;
    long long want = (long long)(per_sm * dev.sms / (double)base + 0.5);
    if (want < 1) want = 1;
    if (small && want < ceil_div(max_tiles, kDecMaxSplitTiles))
      want = ceil_div(max_tiles, kDecMaxSplitTiles);
    tps = (int)ceil_div(max_tiles, want);
    if (tps < 4) tps = 4;
  }
  if (tps > max_tiles && max_tiles > 0) tps = max_tiles;
  // The combine keeps splits x rows weights in shared memory: at most 256 splits.
  if (max_tiles > 0 && ceil_div(max_tiles, tps) > 256) tps = (int)ceil_div(max_tiles, 256);
  pl->tps = tps;
  pl->splits = max_tiles == 0 ? 1 : (int)ceil_div(max_tiles, tps);
  pl->ctas = base * pl->splits;
  if (pl->ctas > 0x7fffffffLL) return GQA_ATTN_ERR_TOO_LARGE;
  if (pl->splits > 1) {
    const size_t prow = (size_t)base * pl->splits * pl->block_rows;
    const size_t o_bytes = align256(prow * pr.d * sizeof(float));
    const size_t lse_bytes = align256(prow * sizeof(float));
    pl->off_lse = o_bytes;
    pl->ws_bytes = o_bytes + lse_bytes;
    pl->ticket_bytes = align256((size_t)base * sizeof(unsigned int));
  }
  return GQA_ATTN_OK;
}

int plan_prefill(const Problem& pr, const DeviceInfo& dev, Plan* pl) {
  pl->path = kPathPrefill;
  pl->dch = pr.d <= 64 ? 1 : 2;
  pl->d_pad = (pr.d + 15) / 16 * 16;
  pl->tiles_per_unit = (int)ceil_div(pr.rows, kPfM);
  pl->pair_heads = (pr.q_len % kPfM == 0 && pr.group % 2 == 0) ? 1 : 0;
  pl->pairs_per_unit = pl->pair_heads ? (pr.group / 2) * (pr.q_len / kPfM)
                                      : (int)ceil_div(pl->tiles_per_unit, 2);
  pl->ctas = pr.units * pl->pairs_per_unit;
  const MaskSpec ms{pr.q_len, pr.kv_len, pr.causal, pr.window};
  int max_tiles = 0;
  for (int t = 0; t < pl->tiles_per_unit; ++t) {
    const long long r0 = (long long)t * kPfM;
    const int nr = (int)((pr.rows - r0) < kPfM ? (pr.rows - r0) : kPfM);
    const KeyRange kr = key_range(ms, r0, nr, kPfN);
    if (kr.t_count > max_tiles) max_tiles = kr.t_count;
  }
  pl->max_tiles = max_tiles;
  // Too few tile pairs to fill the GPU (multi-token decode shapes): split each
  // pair's key range so that about one item per SM runs; the splits' partials
  // are merged by the last split to finish.  Units with a single row tile use
  // both q-tile slots for that tile, on adjacent splits (paired items), so
  // the two softmax warpgroups still alternate.
  pl->splits = 1;
  pl->split_pairs = 0;
  const int forced_splits = g_force_pf_splits.load();
  if (pl->tiles_per_unit == 1 && max_tiles >= 2 && (pr.units < dev.sms || forced_splits > 1)) {
    long long half = forced_splits > 1 ? (forced_splits + 1) / 2 : dev.sms / pr.units;
    if (half > (max_tiles + 1) / 2) half = (max_tiles + 1) / 2;
    if (half < 1) half = 1;
    pl->split_pairs = 1;
    pl->splits = (int)(2 * half);
    pl->pairs_per_unit = 1;
    pl->ctas = pr.units * half;
    // One partial per item (its two splits are combined in the kernel):
    // O as fp32, and (m, l) per column half of the softmax, per row.
    const size_t tiles = (size_t)pr.units;
    pl->ws_bytes = align256(tiles * half * (size_t)pl->d_pad * kPfM * 4);
    pl->off_lse = pl->ws_bytes;
    pl->ws_bytes += align256(tiles * half * 2 * 2 * kPfM * 4);
    // one ticket per (tile, column half)
    pl->ticket_bytes = align256(tiles * 2 * sizeof(unsigned int));
    return GQA_ATTN_OK;
  }
  const long long pairs = pl->ctas;
  if (pairs < dev.sms && max_tiles > 1) {
    long long s = dev.sms / (pairs > 0 ? pairs : 1);
    if (s > max_tiles) s = max_tiles;
    pl->splits = (int)(s < 1 ? 1 : s);
  }
  pl->ctas = pairs * pl->splits;
  if (pl->ctas > 0x7fffffffLL) return GQA_ATTN_ERR_TOO_LARGE;
  if (pl->splits > 1) {
    pl->ws_bytes = align256((size_t)pairs * 2 * pl->splits * (size_t)pl->d_pad * kPfM * 4);
    pl->off_lse = pl->ws_bytes;
    pl->ws_bytes += align256((size_t)pairs * 2 * pl->splits * 2 * 2 * kPfM * 4);
    pl->ticket_bytes = align256((size_t)pairs * 2 * 2 * sizeof(unsigned int));
  }
  return GQA_ATTN_OK;
}

int make_plan(const Problem& pr, const DeviceInfo& dev, Plan* pl) {
  if (pr.batch == 0 || pr.q_len == 0) {
    pl->path = kPathNone;
    return GQA_ATTN_OK;
  }
  if (pr.kv_len == 0) {
    pl->path = kPathZero;
    return GQA_ATTN_OK;
  }
  // Up to 16 rows per kv head (single-token decode) run on the split-KV
  // mma.sync decode kernel; more rows on the tcgen05 kernel (head_dim up to
  // 128), with key-range splits when there are few row tiles; the decode
  // kernel also covers head_dim 136..256.
  const int forced = g_force_path.load();
  // Ring storage is read by the split-KV kernel only.
  const bool prefill_ok = pr.d <= 128 && pr.ring == 0;
  bool prefill = pr.rows > 16 && prefill_ok;
  if (forced == 1) prefill = false;
  if (forced == 2 && prefill_ok) prefill = true;
  return prefill ? plan_prefill(pr, dev, pl) : plan_decode(pr, dev, pl);
}

// ------------------------------------------------------------------ workspace
struct Workspace {
  void* ptr = nullptr;
  size_t bytes = 0;
  void* tickets = nullptr;
  size_t ticket_bytes = 0;
};
std::map<std::pair<int, cudaStream_t>, Workspace> g_ws;
// Buffers replaced by bigger ones: kept, not freed, because a CUDA graph
// captured earlier may still reference them (freed by
// gqa_attn_release_workspace).  Tickets are listed with their size so that
// gqa_attn_clear_status can zero them too.
struct Retired {
  int dev;
  void* ptr;
  size_t ticket_bytes;  // > 0: a ticket buffer
};
std::vector<Retired> g_retired;

// Workspace for (current device, stream): `bytes` of scratch for the split
// partials and `ticket_bytes` of ticket counters.  Tickets live in their own
// buffer, cleared on allocation; every kernel leaves its tickets at zero.
// Growing allocates new buffers (no synchronisation) and retires the old.
int get_workspace(cudaStream_t stream, size_t bytes, size_t ticket_bytes, void** out,
                  void** tickets) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GQA_ATTN_ERR_DEVICE;
  std::lock_guard<std::mutex> lk(g_mu);
  Workspace& ws = g_ws[std::make_pair(dev, stream)];
  if (ws.bytes < bytes) {
    void* p = nullptr;
    const size_t want = bytes + bytes / 4;
    if (cudaMalloc(&p, want) != cudaSuccess) {
      cudaGetLastError();
      return GQA_ATTN_ERR_ALLOC;
    }
    if (ws.ptr) g_retired.push_back({dev, ws.ptr, 0});
    ws.ptr = p;
    ws.bytes = want;
  }
  if (ws.ticket_bytes < ticket_bytes) {
    void* p = nullptr;
    const size_t want = ticket_bytes < 4096 ? 4096 : ticket_bytes * 2;
    if (cudaMalloc(&p, want) != cudaSuccess) {
      cudaGetLastError();
      return GQA_ATTN_ERR_ALLOC;
    }
    if (cudaMemsetAsync(p, 0, want, stream) != cudaSuccess) {
      cudaFree(p);
      return GQA_ATTN_ERR_LAUNCH;
    }
    if (ws.tickets) g_retired.push_back({dev, ws.tickets, ws.ticket_bytes});
    ws.tickets = p;
    ws.ticket_bytes = want;
  }
  *out = ws.ptr;
  *tickets = ws.tickets;
  return GQA_ATTN_OK;
}

// ------------------------------------------------------------------ TMA maps
// 4-D bf16 view of K or V: (col < d, key < kv_len, kv head, batch) over
// either cache layout, with a (64 cols x box_rows x 1 x 1) box, 128-byte
// swizzle; keys at or past kv_len read as zero.
int encode_kv_map(CUtensorMap* map, const void* base, const Problem& pr, int box_rows) {
  const cuuint64_t e = 2, d = (cuuint64_t)pr.d, h = (cuuint64_t)pr.hkv,
                   s = (cuuint64_t)pr.kv_alloc;
  // A ring's map covers all its slots; keys in order stop at kv_len.
  const cuuint64_t rows = pr.ring ? (cuuint64_t)pr.ring : (cuuint64_t)pr.kv_len;
  cuuint64_t dims[4] = {d, rows, h, (cuuint64_t)pr.batch};
  cuuint64_t strides[3];
  if (pr.kv_seq_major) {
    strides[0] = h * d * e;      // next key
    strides[1] = d * e;          // next head
  } else {
    strides[0] = d * e;
    strides[1] = s * d * e;
  }
  strides[2] = s * h * d * e;    // next batch element
  cuuint32_t box[4] = {64, (cuuint32_t)box_rows, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    snprintf(g_detail, sizeof g_detail, "cuTensorMapEncodeTiled (k/v): CUresult %d", (int)r);
    return GQA_ATTN_ERR_LAUNCH;
  }
  return GQA_ATTN_OK;
}

// 3-D bf16 view [outer][rows][cols] with a (64 cols x box_rows x 1) box,
// 128-byte swizzle; out-of-range elements read as zero.
int encode_map(CUtensorMap* map, const void* base, int cols, long long rows, long long outer,
               int box_rows) {
  cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)outer};
  cuuint64_t strides[2] = {(cuuint64_t)cols * 2, (cuuint64_t)cols * 2 * (cuuint64_t)rows};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    snprintf(g_detail, sizeof g_detail, "cuTensorMapEncodeTiled: CUresult %d", (int)r);
    return GQA_ATTN_ERR_LAUNCH;
  }
  return GQA_ATTN_OK;
}

// ------------------------------------------------------------------ launches
template <int KS, bool kT, bool kDeep = false>
int launch_decode_ks(const Problem& pr, const Plan& pl, DeviceInfo& dev, const void* q,
                     const void* k, const void* v, void* o, void* ws, void* tickets,
                     cudaStream_t stream) {
  using C = DecodeCfg<KS, kDeep>;
  const int slot = kDeep ? 8 + (KS / 4 - 1) : (KS / 4 - 1) + (kT ? 4 : 0);
  std::unique_lock<std::mutex> lk(g_mu);
  if (!dev.decode_attr[slot]) {
    cudaError_t e = cudaFuncSetAttribute(decode_splitkv_kernel<KS, kT, kDeep>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::kSmemBytes);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(decode_splitkv_kernel<KS, kT, kDeep>,
                               cudaFuncAttributePreferredSharedMemoryCarveout,
                               cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return cuda_fail("cudaFuncSetAttribute(decode)", e, GQA_ATTN_ERR_LAUNCH);
    dev.decode_attr[slot] = true;
  }
  lk.unlock();
  CUtensorMap tk, tv;
  if (encode_kv_map(&tk, k, pr, kDecTile) != GQA_ATTN_OK ||
      encode_kv_map(&tv, v, pr, kDecTile) != GQA_ATTN_OK)
    return GQA_ATTN_ERR_LAUNCH;
  DecodeParams p;
  p.q = (const __nv_bfloat16*)q;
  p.o = (__nv_bfloat16*)o;
  p.q_len = pr.q_len;
  p.kv_len = pr.kv_len;
  p.kv_heads = pr.hkv;
  p.k_base = pr.ring ? ring_k_base(pr.kv_len, pr.ring, kDecTile) : 0;
  p.ring_tiles = pr.ring ? pr.ring / kDecTile : 0;
  p.ring_phase = pr.ring ? ring_phase(pr.kv_len, pr.ring, kDecTile) : 0;
  p.app_count = pr.app_count;
  p.app_pos = pr.app_pos;
  p.app_slots = (int)pr.kv_alloc;
  p.app_ring = pr.ring ? 1 : 0;
  p.app_new_f32 = pr.app_new_f32;
  p.app_new_head_major = pr.app_new_head_major;
  p.app_cache_seq_major = pr.kv_seq_major;
  p.app_new_k = pr.app_new_k;
  p.app_new_v = pr.app_new_v;
  p.app_k_cache = (__nv_bfloat16*)k;
  p.app_v_cache = (__nv_bfloat16*)v;
  p.head_dim = pr.d;
  p.rows = (int)pr.rows;
  p.row_blocks = pl.row_blocks;
  p.block_rows = pl.block_rows;
  p.causal = pr.causal;
  p.window = pr.window;
  p.use_softcap = pr.softcap > 0.f ? 1 : 0;
  const float rs = 1.0f / std::sqrt((float)pr.d);
  p.logit_scale = kLog2e * rs;
  p.cap_in = p.use_softcap ? rs / pr.softcap : 0.f;
  p.cap_out = p.use_softcap ? pr.softcap * kLog2e : 0.f;
  p.splits = pl.splits;
  p.tiles_per_split = pl.tps;
  p.part_o = (float*)ws;
  p.part_lse = ws ? (float*)((char*)ws + pl.off_lse) : nullptr;
  p.tickets = (unsigned int*)tickets;
  decode_splitkv_kernel<KS, kT, kDeep>
      <<<dim3((unsigned)pl.ctas), kDecThreads, C::kSmemBytes, stream>>>(tk, tv, p);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? GQA_ATTN_OK : cuda_fail("launch(decode)", e, GQA_ATTN_ERR_LAUNCH);
}

int launch_decode(const Problem& pr, const Plan& pl, DeviceInfo& dev, const void* q,
                  const void* k, const void* v, void* o, void* ws, void* tickets,
                  cudaStream_t stream) {
  if (pl.block_rows <= 8) {  // single-token decode shapes: keys-as-M variant
    // At most one CTA per SM: the deeper ring keeps more bytes in flight.
    const bool deep = pl.ctas <= dev.sms;
    switch (pl.ks) {
      case 4:
        return deep ? launch_decode_ks<4, true, true>(pr, pl, dev, q, k, v, o, ws, tickets, stream)
                    : launch_decode_ks<4, true>(pr, pl, dev, q, k, v, o, ws, tickets, stream);
      case 8:
        return deep ? launch_decode_ks<8, true, true>(pr, pl, dev, q, k, v, o, ws, tickets, stream)
                    : launch_decode_ks<8, true>(pr, pl, dev, q, k, v, o, ws, tickets, stream);
      case 12: return launch_decode_ks<12, true>(pr, pl, dev, q, k, v, o, ws, tickets, stream);
      default: return launch_decode_ks<16, true>(pr, pl, dev, q, k, v, o, ws, tickets, stream);
    }
  }
  switch (pl.ks) {
    case 4: return launch_decode_ks<4, false>(pr, pl, dev, q, k, v, o, ws, tickets, stream);
    case 8: return launch_decode_ks<8, false>(pr, pl, dev, q, k, v, o, ws, tickets, stream);
    case 12: return launch_decode_ks<12, false>(pr, pl, dev, q, k, v, o, ws, tickets, stream);
    default: return launch_decode_ks<16, false>(pr, pl, dev, q, k, v, o, ws, tickets, stream);
  }
}

// Exponent-base offset B of the fixed-base softcap path for this cap (in
// log2 units, cap_out = softcap * log2 e): B = max(16, 2 cap_out - 120), used
// only when B <= 64 (see PrefillParams::cap_fixed).
float cap_base_offset(float cap_out) { return std::max(16.0f, 2.0f * cap_out - 120.0f); }

// Softcap code of the tcgen05 kernel: 0 = no softcap; 3 = the degree-5
// tanh polynomial with a fixed exponent base (no row max; caps up to about
// 63.8); 5 = the degree-5 polynomial with the row max (caps up to
// kTanh5MaxCap, or any cap when override key 5 asks for it); 7 = degree 7.
int cap_degree(const Problem& pr) {
  if (!(pr.softcap > 0.f)) return 0;
  if (pr.softcap > kTanh5MaxCap) return 7;
  const bool fixed = cap_base_offset(pr.softcap * kLog2e) <= 64.0f && g_force_two_pass.load() == 0;
  return fixed ? 3 : 5;
}

// kSplit: 0 = no key splits, 1 = splits merged through the workspace,
// 2 = paired splits merged inside a cluster.
template <int DCH, int kCapDeg, int kSplit>
constexpr int prefill_slot() {
  return (DCH - 1) + 2 * (kCapDeg == 5 ? 1 : kCapDeg == 7 ? 2 : kCapDeg == 3 ? 3 : 0) +
         8 * kSplit;
}

// One-time per device and instantiation (under g_mu): the register-split
// check and the dynamic shared memory limit.
template <int DCH, int kCapDeg, int kSplit>
int prefill_setup(DeviceInfo& dev) {
  using C = PrefillCfg<DCH>;
  constexpr int attr = prefill_slot<DCH, kCapDeg, kSplit>();
  std::lock_guard<std::mutex> lk(g_mu);
  if (dev.prefill_attr[attr]) return GQA_ATTN_OK;
  // The register split inside the kernel must fit what the block is
  // launched with, or setmaxnreg.inc could never be granted.
  cudaFuncAttributes fa;
  const cudaError_t ea = cudaFuncGetAttributes(&fa, prefill_sm100_kernel<DCH, kCapDeg, kSplit>);
  if (ea != cudaSuccess) return cuda_fail("cudaFuncGetAttributes(prefill)", ea, GQA_ATTN_ERR_LAUNCH);
  if ((long long)fa.numRegs * kPfThreads < kRegSplitTotal) {
    snprintf(g_detail, sizeof g_detail, "prefill kernel built with %d registers/thread: "
             "register split needs %d", fa.numRegs, kRegSplitTotal);
    return GQA_ATTN_ERR_LAUNCH;
  }
  const cudaError_t e = cudaFuncSetAttribute(prefill_sm100_kernel<DCH, kCapDeg, kSplit>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::kSmemBytes);
  if (e != cudaSuccess) return cuda_fail("cudaFuncSetAttribute(prefill)", e, GQA_ATTN_ERR_LAUNCH);
  dev.prefill_attr[attr] = true;
  return GQA_ATTN_OK;
}

// Paired key splits, one item per CTA: a cluster per unit merges its
// partials (every CTA a column slice, after the cluster barrier) when every
// cluster of the grid can be resident at once (one wave) and a unit has 2..8
// CTAs; *csize gets the CTAs per cluster, or 0 for the merge by the last CTA
// of a unit (ticket).
template <int DCH, int kCapDeg>
int prefill_cluster_k(const Problem& pr, const Plan& pl, DeviceInfo& dev, int* csize) {
  using C = PrefillCfg<DCH>;
  *csize = 0;
  if (!pl.split_pairs || g_no_cluster.load()) return GQA_ATTN_OK;
  const int half = pl.splits / 2;
  if (half < 2 || half > 8 || pl.ctas != pr.units * half) return GQA_ATTN_OK;
  int rc = prefill_setup<DCH, kCapDeg, 2>(dev);
  if (rc != GQA_ATTN_OK) return rc;
  constexpr int attr = prefill_slot<DCH, kCapDeg, 2>();
  std::lock_guard<std::mutex> lk(g_mu);
  int& fit = dev.cluster_max[attr][half];
  if (fit < 0) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = (unsigned)half;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3((unsigned)pl.ctas);
    cfg.blockDim = dim3(kPfThreads);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, prefill_sm100_kernel<DCH, kCapDeg, 2>, &cfg) !=
        cudaSuccess) {
      (void)cudaGetLastError();
      n = 0;
    }
    fit = n;
  }
  if (fit >= pr.units) *csize = half;
  return GQA_ATTN_OK;
}

int prefill_cluster(const Problem& pr, const Plan& pl, DeviceInfo& dev, int* csize) {
  const int deg = cap_degree(pr);
  if (pl.dch == 1)
    return deg == 3 ? prefill_cluster_k<1, 3>(pr, pl, dev, csize)
         : deg == 5 ? prefill_cluster_k<1, 5>(pr, pl, dev, csize)
         : deg == 7 ? prefill_cluster_k<1, 7>(pr, pl, dev, csize)
                    : prefill_cluster_k<1, 0>(pr, pl, dev, csize);
  return deg == 3 ? prefill_cluster_k<2, 3>(pr, pl, dev, csize)
       : deg == 5 ? prefill_cluster_k<2, 5>(pr, pl, dev, csize)
       : deg == 7 ? prefill_cluster_k<2, 7>(pr, pl, dev, csize)
                  : prefill_cluster_k<2, 0>(pr, pl, dev, csize);
}

template <int DCH, int kCapDeg, int kSplit>
int launch_prefill_k(const Problem& pr, const Plan& pl, DeviceInfo& dev, int csize,
                     const void* q, const void* k, const void* v, void* o, void* ws,
                     void* tickets, cudaStream_t stream) {
  using C = PrefillCfg<DCH>;
  constexpr bool kCap = kCapDeg != 0;
  int rc = prefill_setup<DCH, kCapDeg, kSplit>(dev);
  if (rc != GQA_ATTN_OK) return rc;
  CUtensorMap tq, tk, tv, to;
  if (encode_map(&tq, q, pr.d, pr.rows, pr.units, kPfM) != GQA_ATTN_OK ||
      encode_map(&to, o, pr.d, pr.rows, pr.units, 32) != GQA_ATTN_OK ||
      encode_kv_map(&tk, k, pr, kPfN) != GQA_ATTN_OK ||
      encode_kv_map(&tv, v, pr, kPfN) != GQA_ATTN_OK)
    return GQA_ATTN_ERR_LAUNCH;
  PrefillParams p;
  p.o = (__nv_bfloat16*)o;
  p.q_len = pr.q_len;
  p.kv_len = pr.kv_len;
  p.kv_heads = pr.hkv;
  p.head_dim = pr.d;
  p.d_pad = pl.d_pad;
  p.rows = (int)pr.rows;
  p.tiles_per_unit = pl.tiles_per_unit;
  p.pairs_per_unit = pl.pairs_per_unit;
  p.splits = pl.splits;
  p.split_pairs = pl.split_pairs;
  p.n_items = (int)pl.ctas;
  p.ws_o = (float*)ws;
  p.ws_ml = ws ? (float*)((char*)ws + pl.off_lse) : nullptr;
  p.tickets = (unsigned int*)tickets;
  p.pair_heads = pl.pair_heads;
  p.heavy_first = (pr.causal || pr.window > 0) && !pl.split_pairs ? 1 : 0;
  p.cluster_merge = kSplit == 2 ? csize : 0;
  p.causal = pr.causal;
  p.window = pr.window;
  const float rs = 1.0f / std::sqrt((float)pr.d);
  p.logit_scale = kLog2e * rs;
  p.cap_in = kCap ? rs / pr.softcap : 0.f;
  p.cap_out = kCap ? pr.softcap * kLog2e : 0.f;
  // Fixed exponent base (softcap code 3, see PrefillParams and cap_degree).
  p.cap_fixed = kCapDeg == 3 ? 1 : 0;
  p.cap_base = kCapDeg == 3 ? p.cap_out - cap_base_offset(p.cap_out) : 0.f;
  if constexpr (kSplit == 2) {
    // One item per CTA, clusters of csize consecutive CTAs (one unit each).
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = (unsigned)csize;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3((unsigned)pl.ctas);
    cfg.blockDim = dim3(kPfThreads);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = stream;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    const cudaError_t e =
        cudaLaunchKernelEx(&cfg, prefill_sm100_kernel<DCH, kCapDeg, kSplit>, tq, tk, tv, to, p);
    return e == cudaSuccess ? GQA_ATTN_OK : cuda_fail("launch(prefill, clusters)", e, GQA_ATTN_ERR_LAUNCH);
  }
  // Persistent: at most one CTA per SM, each walking items with stride grid.
  const int grid = (int)(pl.ctas < dev.sms ? pl.ctas : dev.sms);
  prefill_sm100_kernel<DCH, kCapDeg, kSplit><<<dim3((unsigned)grid), kPfThreads, C::kSmemBytes, stream>>>(
      tq, tk, tv, to, p);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? GQA_ATTN_OK : cuda_fail("launch(prefill)", e, GQA_ATTN_ERR_LAUNCH);
}

template <int DCH, int kCapDeg>
int launch_prefill_d(const Problem& pr, const Plan& pl, DeviceInfo& dev, int csize,
                     const void* q, const void* k, const void* v, void* o, void* ws,
                     void* tickets, cudaStream_t stream) {
  if (pl.splits <= 1)
    return launch_prefill_k<DCH, kCapDeg, 0>(pr, pl, dev, csize, q, k, v, o, ws, tickets, stream);
  if (csize > 0)
    return launch_prefill_k<DCH, kCapDeg, 2>(pr, pl, dev, csize, q, k, v, o, ws, tickets, stream);
  return launch_prefill_k<DCH, kCapDeg, 1>(pr, pl, dev, csize, q, k, v, o, ws, tickets, stream);
}

int launch_prefill(const Problem& pr, const Plan& pl, DeviceInfo& dev, int csize, const void* q,
                   const void* k, const void* v, void* o, void* ws, void* tickets,
                   cudaStream_t stream) {
  const int deg = cap_degree(pr);
  if (pl.dch == 1)
    return deg == 3 ? launch_prefill_d<1, 3>(pr, pl, dev, csize, q, k, v, o, ws, tickets, stream)
         : deg == 5 ? launch_prefill_d<1, 5>(pr, pl, dev, csize, q, k, v, o, ws, tickets, stream)
         : deg == 7 ? launch_prefill_d<1, 7>(pr, pl, dev, csize, q, k, v, o, ws, tickets, stream)
                    : launch_prefill_d<1, 0>(pr, pl, dev, csize, q, k, v, o, ws, tickets, stream);
  return deg == 3 ? launch_prefill_d<2, 3>(pr, pl, dev, csize, q, k, v, o, ws, tickets, stream)
       : deg == 5 ? launch_prefill_d<2, 5>(pr, pl, dev, csize, q, k, v, o, ws, tickets, stream)
       : deg == 7 ? launch_prefill_d<2, 7>(pr, pl, dev, csize, q, k, v, o, ws, tickets, stream)
                  : launch_prefill_d<2, 0>(pr, pl, dev, csize, q, k, v, o, ws, tickets, stream);
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  if (!a || !b || na == 0 || nb == 0) return false;
  const uintptr_t x = (uintptr_t)a, y = (uintptr_t)b;
  return x < y + nb && y < x + na;
}

// Ring storage of `slots` slots (key j in slot j % slots): the slots must
// be whole 64-key tiles and hold every key any query can see, i.e. the
// keys from kv_len - slots on (the window bounds how far back queries look).
int set_ring(Problem* pr, int slots) {
  if (slots <= 0 || slots % kDecTile != 0) return GQA_ATTN_ERR_ARG;
  long long reach;  // keys back from kv_len that the oldest query may see
  if (pr->window > 0)
    reach = (long long)pr->q_len + pr->window - 1;
  else
    reach = pr->kv_len;
  if (reach > pr->kv_len) reach = pr->kv_len;
  if (reach > slots) {
    snprintf(g_detail, sizeof g_detail, "ring of %d slots holds fewer keys than the %lld visible",
             slots, reach);
    return GQA_ATTN_ERR_ARG;
  }
  pr->ring = slots;
  pr->kv_alloc = slots;
  return GQA_ATTN_OK;
}

int check_pointers(const Problem& pr, const void* q, const void* k, const void* v,
                   const void* o) {
  const size_t q_bytes = (size_t)pr.batch * pr.hq * (size_t)pr.q_len * pr.d * 2;
  const size_t kv_bytes = (size_t)pr.batch * pr.hkv * (size_t)pr.kv_alloc * pr.d * 2;
  if (q_bytes && (!q || !o)) return GQA_ATTN_ERR_NULL_POINTER;
  if (kv_bytes && (!k || !v)) return GQA_ATTN_ERR_NULL_POINTER;
  if (((uintptr_t)q | (uintptr_t)k | (uintptr_t)v | (uintptr_t)o) & 15u)
    return GQA_ATTN_ERR_MISALIGNED;
  if (overlaps(o, q_bytes, q, q_bytes) || overlaps(o, q_bytes, k, kv_bytes) ||
      overlaps(o, q_bytes, v, kv_bytes))
    return GQA_ATTN_ERR_ALIAS;
  return GQA_ATTN_OK;
}

int run(const Problem& pr, const void* q, const void* k, const void* v, void* o,
        cudaStream_t stream) {
  DeviceInfo* dev = nullptr;
  int rc = device_info(&dev);
  if (rc != GQA_ATTN_OK) return rc;
  Plan pl;
  rc = make_plan(pr, *dev, &pl);
  if (rc != GQA_ATTN_OK) return rc;
  switch (pl.path) {
    case kPathNone:
      return GQA_ATTN_OK;
    case kPathZero: {
      const size_t bytes = (size_t)pr.batch * pr.hq * (size_t)pr.q_len * pr.d * 2;
      return cudaMemsetAsync(o, 0, bytes, stream) == cudaSuccess ? GQA_ATTN_OK
                                                                 : GQA_ATTN_ERR_LAUNCH;
    }
    default: {
      // Key splits merge through the workspace: by the last CTA of a unit to
      // finish (ticket), or by all CTAs of the unit's cluster together.
      int csize = 0;
      if (pl.path == kPathPrefill && pl.splits > 1) {
        rc = prefill_cluster(pr, pl, *dev, &csize);
        if (rc != GQA_ATTN_OK) return rc;
      }
      void* ws = nullptr;
      void* tickets = nullptr;
      if (pl.ws_bytes) {
        rc = get_workspace(stream, pl.ws_bytes, pl.ticket_bytes, &ws, &tickets);
        if (rc != GQA_ATTN_OK) return rc;
      }
      if (pl.path == kPathPrefill)
        return launch_prefill(pr, pl, *dev, csize, q, k, v, o, ws, tickets, stream);
      return launch_decode(pr, pl, *dev, q, k, v, o, ws, tickets, stream);
    }
  }
}

// ------------------------------------------------------------------ static scratch
// Scratch for gqa_attn_fwd_static_scratch: a fixed array in device memory,
// created with the module on every GPU that loads this library and kept
// until the process exits.  Layout: [0, kStaticTicketBytes) split tickets,
// then the split partials (o_s, then lse_s).  Host code must not pass the
// array's name to a kernel (in host code it is only a stand-in for the
// symbol); its device address comes from cudaGetSymbolAddress below.
constexpr size_t kStaticScratchBytes = 8u << 20;  // 8 MiB
constexpr size_t kStaticTicketBytes = 64u << 10;  // 16384 tickets
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

void* g_static_scratch_addr[64] = {};

// Device address of g_static_scratch on the current device, looked up once
// per device (with that device current) and cached.
int static_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return GQA_ATTN_ERR_DEVICE;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_static_scratch_addr[dev]) {
    void* ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_static_scratch);
    if (e != cudaSuccess || ptr == nullptr)
      return cuda_fail("cudaGetSymbolAddress(g_static_scratch)", e, GQA_ATTN_ERR_LAUNCH);
    g_static_scratch_addr[dev] = ptr;
  }
  *out = g_static_scratch_addr[dev];
  return GQA_ATTN_OK;
}

}  // namespace

// ==================================================================== C ABI
extern "C" {

int gqa_attn_fwd(const void* q, const void* k, const void* v, void* o, int batch, int q_len,
                 int kv_len, int num_q_heads, int num_kv_heads, int head_dim, int causal,
                 int window, float softcap, void* stream) {
  Problem pr;
  int rc = validate(batch, q_len, kv_len, num_q_heads, num_kv_heads, head_dim, causal, window,
                    softcap, &pr);
  if (rc != GQA_ATTN_OK) return rc;
  rc = check_pointers(pr, q, k, v, o);
  if (rc != GQA_ATTN_OK) return rc;
  return run(pr, q, k, v, o, (cudaStream_t)stream);
}

int gqa_attn_fwd_host(const void* q_host, const void* k_host, const void* v_host, void* o_host,
                      void* q_dev, void* k_dev, void* v_dev, void* o_dev, int batch, int q_len,
                      int kv_len, int num_q_heads, int num_kv_heads, int head_dim, int causal,
                      int window, float softcap, void* stream) {
  Problem pr;
  int rc = validate(batch, q_len, kv_len, num_q_heads, num_kv_heads, head_dim, causal, window,
                    softcap, &pr);
  if (rc != GQA_ATTN_OK) return rc;
  rc = check_pointers(pr, q_dev, k_dev, v_dev, o_dev);
  if (rc != GQA_ATTN_OK) return rc;
  const size_t q_bytes = (size_t)pr.batch * pr.hq * (size_t)pr.q_len * pr.d * 2;
  const size_t kv_bytes = (size_t)pr.batch * pr.hkv * (size_t)pr.kv_len * pr.d * 2;
  if ((q_bytes && (!q_host || !o_host)) || (kv_bytes && (!k_host || !v_host)))
    return GQA_ATTN_ERR_NULL_POINTER;
  cudaStream_t s = (cudaStream_t)stream;
  if (q_bytes && cudaMemcpyAsync(q_dev, q_host, q_bytes, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return GQA_ATTN_ERR_LAUNCH;
  if (kv_bytes &&
      (cudaMemcpyAsync(k_dev, k_host, kv_bytes, cudaMemcpyHostToDevice, s) != cudaSuccess ||
       cudaMemcpyAsync(v_dev, v_host, kv_bytes, cudaMemcpyHostToDevice, s) != cudaSuccess))
    return GQA_ATTN_ERR_LAUNCH;
  rc = run(pr, q_dev, k_dev, v_dev, o_dev, s);
  if (rc != GQA_ATTN_OK) return rc;
  if (q_bytes && cudaMemcpyAsync(o_host, o_dev, q_bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return GQA_ATTN_ERR_LAUNCH;
  return cudaStreamSynchronize(s) == cudaSuccess ? GQA_ATTN_OK : GQA_ATTN_ERR_LAUNCH;
}

int gqa_attn_describe(int batch, int q_len, int kv_len, int num_q_heads, int num_kv_heads,
                      int head_dim, int causal, int window, float softcap, int* path, int* splits,
                      int* ctas, int* tiles) {
  Problem pr;
  int rc = validate(batch, q_len, kv_len, num_q_heads, num_kv_heads, head_dim, causal, window,
                    softcap, &pr);
  if (rc != GQA_ATTN_OK) return rc;
  DeviceInfo* dev = nullptr;
  rc = device_info(&dev);
  if (rc != GQA_ATTN_OK) return rc;
  Plan pl;
  rc = make_plan(pr, *dev, &pl);
  if (rc != GQA_ATTN_OK) return rc;
  if (path) *path = pl.path;
  if (splits) *splits = pl.splits;
  if (ctas) *ctas = (int)pl.ctas;
  if (tiles) *tiles = pl.max_tiles;
  return GQA_ATTN_OK;
}

int gqa_attn_set_override(int key, int value) {
  if (key == 1) {
    g_force_path.store(value);
    return GQA_ATTN_OK;
  }
  if (key == 2) {
    g_force_tps.store(value > 0 ? value : 0);
    return GQA_ATTN_OK;
  }
  if (key == 3) {
    g_force_pf_splits.store(value > 0 ? value : 0);
    return GQA_ATTN_OK;
  }
  if (key == 4) {
    g_no_cluster.store(value < 0 ? 1 : 0);
    return GQA_ATTN_OK;
  }
  if (key == 5) {
    g_force_two_pass.store(value ? 1 : 0);
    return GQA_ATTN_OK;
  }
  return GQA_ATTN_ERR_ARG;
}

const char* gqa_attn_error_string(int status) {
  switch (status) {
    case GQA_ATTN_OK: return "ok";
    case GQA_ATTN_ERR_NULL_POINTER: return "null pointer for a tensor with elements";
    case GQA_ATTN_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case GQA_ATTN_ERR_BAD_SHAPE: return "invalid size (negative, or zero heads)";
    case GQA_ATTN_ERR_HEAD_RATIO: return "num_q_heads is not a multiple of num_kv_heads";
    case GQA_ATTN_ERR_HEAD_DIM: return "head_dim must be a multiple of 8 in [8, 256]";
    case GQA_ATTN_ERR_SOFTCAP: return "softcap must be finite and >= 0";
    case GQA_ATTN_ERR_DEVICE: return "current device is not an sm_100 (B200-class) GPU";
    case GQA_ATTN_ERR_LAUNCH: return "CUDA launch or copy failed";
    case GQA_ATTN_ERR_ALLOC: return "workspace allocation failed";
    case GQA_ATTN_ERR_TOO_LARGE: return "problem exceeds the kernels' index range";
    case GQA_ATTN_ERR_ALIAS: return "output overlaps an input";
    case GQA_ATTN_ERR_ARG: return "invalid argument";
    default: return "unknown status";
  }
}

int gqa_attn_status(void) {
  uint32_t v = 0;
  if (cudaMemcpyFromSymbol(&v, gqa::g_gqa_status, sizeof v) != cudaSuccess) return -1;
  return (int)v;
}

int gqa_attn_clear_status(void) {
  const uint32_t z = 0;
  if (cudaMemcpyToSymbol(gqa::g_gqa_status, &z, sizeof z) != cudaSuccess) return GQA_ATTN_ERR_LAUNCH;
  // A kernel that gave up a wait may have left split tickets counted, which
  // would make the next merge on that buffer start early or never: zero
  // every ticket buffer of this device (active and retired).
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GQA_ATTN_ERR_DEVICE;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    for (auto& kv : g_ws)
      if (kv.first.first == dev && kv.second.tickets &&
          cudaMemset(kv.second.tickets, 0, kv.second.ticket_bytes) != cudaSuccess)
        return GQA_ATTN_ERR_LAUNCH;
    for (const Retired& r : g_retired)
      if (r.dev == dev && r.ticket_bytes > 0 && cudaMemset(r.ptr, 0, r.ticket_bytes) != cudaSuccess)
        return GQA_ATTN_ERR_LAUNCH;
  }
  return cudaDeviceSynchronize() == cudaSuccess ? GQA_ATTN_OK : GQA_ATTN_ERR_LAUNCH;
}

int gqa_attn_release_workspace(void) {
  int cur = 0;
  if (cudaGetDevice(&cur) != cudaSuccess) return GQA_ATTN_ERR_DEVICE;
  std::lock_guard<std::mutex> lk(g_mu);
  int rc = GQA_ATTN_OK;
  auto release = [&](int dev, void* p) {
    if (!p) return;
    if (cudaSetDevice(dev) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess ||
        cudaFree(p) != cudaSuccess)
      rc = GQA_ATTN_ERR_LAUNCH;
  };
  for (auto& kv : g_ws) {
    release(kv.first.first, kv.second.ptr);
    release(kv.first.first, kv.second.tickets);
  }
  g_ws.clear();
  for (const Retired& r : g_retired) release(r.dev, r.ptr);
  g_retired.clear();
  if (cudaSetDevice(cur) != cudaSuccess) rc = GQA_ATTN_ERR_DEVICE;
  return rc;
}

int gqa_attn_describe_merge(int batch, int q_len, int kv_len, int num_q_heads, int num_kv_heads,
                            int head_dim, int causal, int window, float softcap, int* cluster) {
  Problem pr;
  int rc = validate(batch, q_len, kv_len, num_q_heads, num_kv_heads, head_dim, causal, window,
                    softcap, &pr);
  if (rc != GQA_ATTN_OK) return rc;
  DeviceInfo* dev = nullptr;
  rc = device_info(&dev);
  if (rc != GQA_ATTN_OK) return rc;
  Plan pl;
  rc = make_plan(pr, *dev, &pl);
  if (rc != GQA_ATTN_OK) return rc;
  int csize = 0;
  if (pl.path == kPathPrefill && pl.splits > 1) {
    rc = prefill_cluster(pr, pl, *dev, &csize);
    if (rc != GQA_ATTN_OK) return rc;
  }
  if (cluster) *cluster = csize;
  return GQA_ATTN_OK;
}

int gqa_attn_selftest_bounded_wait(int limit_us, void* stream) {
  if (limit_us < 1 || limit_us > 10000000) return GQA_ATTN_ERR_ARG;
  DeviceInfo* dev = nullptr;
  int rc = device_info(&dev);
  if (rc != GQA_ATTN_OK) return rc;
  gqa::selftest_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>((unsigned long long)limit_us *
                                                                 1000ull);
  return cudaGetLastError() == cudaSuccess ? GQA_ATTN_OK : GQA_ATTN_ERR_LAUNCH;
}

int gqa_attn_version(void) { return 300; }

// Argument checks of a KV-cache append (nothing launched).  *n_out gets the
// number of new elements per tensor; GQA_ATTN_OK with *n_out == 0 means
// there is nothing to write.
static int append_checks(void* k_cache, void* v_cache, const void* new_k, const void* new_v,
                         int batch, int cache_slots, int num_kv_heads, int head_dim,
                         int position, int count, unsigned int flags, long long* n_out) {
  *n_out = 0;
  if (flags & ~(GQA_KV_CACHE_SEQ_MAJOR | GQA_KV_CACHE_F32 | GQA_KV_NEW_BF16 |
                GQA_KV_NEW_HEAD_MAJOR | GQA_KV_RING))
    return GQA_ATTN_ERR_ARG;
  if (batch < 0 || num_kv_heads < 1 || cache_slots < 0 || count < 0)
    return GQA_ATTN_ERR_BAD_SHAPE;
  if (head_dim < 8 || head_dim > 256 || head_dim % 8 != 0) return GQA_ATTN_ERR_HEAD_DIM;
  const bool ring = (flags & GQA_KV_RING) != 0;
  if (position < 0 || (long long)position + count > (ring ? 0x7fffffffLL : (long long)cache_slots) ||
      (ring && count > cache_slots))
    return GQA_ATTN_ERR_ARG;
  const long long n = (long long)batch * num_kv_heads * count * head_dim;
  if (n == 0) return GQA_ATTN_OK;
  if (2 * n / 8 + 4LL * 8 * 1024 * 256 >= (1LL << 32)) {  // chunk indices are 32-bit
    snprintf(g_detail, sizeof g_detail, "kv_append: %lld new elements exceed the 32-bit index",
             n);
    return GQA_ATTN_ERR_TOO_LARGE;
  }
  if (!k_cache || !v_cache || !new_k || !new_v) return GQA_ATTN_ERR_NULL_POINTER;
  if (((uintptr_t)k_cache | (uintptr_t)v_cache | (uintptr_t)new_k | (uintptr_t)new_v) & 15u)
    return GQA_ATTN_ERR_MISALIGNED;
  const size_t cache_bytes = (size_t)batch * num_kv_heads * (size_t)cache_slots * head_dim *
                             ((flags & GQA_KV_CACHE_F32) ? 4 : 2);
  const size_t new_bytes = (size_t)n * ((flags & GQA_KV_NEW_BF16) ? 2 : 4);
  if (overlaps(k_cache, cache_bytes, v_cache, cache_bytes) ||
      overlaps(new_k, new_bytes, k_cache, cache_bytes) ||
      overlaps(new_k, new_bytes, v_cache, cache_bytes) ||
      overlaps(new_v, new_bytes, k_cache, cache_bytes) ||
      overlaps(new_v, new_bytes, v_cache, cache_bytes))
    return GQA_ATTN_ERR_ALIAS;
  *n_out = n;
  return GQA_ATTN_OK;
}

// The staged-runs kernel applies when the source and the cache share their
// layout (so one batch row, or one (batch, head) row, of new tokens is one
// contiguous run in both), a ring does not wrap inside the block, and the
// block is large enough for whole chunks to pay off (runs of at least 1024
// elements, a million elements per tensor) but its runs stay below 2^31
// elements; small appends (a decode step) keep the generic kernel.
static bool append_runs_eligible(const KvAppendParams& p, long long n) {
  if (p.cache_seq_major == p.new_head_major) return false;
  const long long slot0 = p.ring ? (long long)p.position % p.slots : p.position;
  if (slot0 + p.count > p.slots) return false;
  const long long run_len =
      p.cache_seq_major ? (long long)p.count * p.heads * p.head_dim : (long long)p.count * p.head_dim;
  // Run lengths and chunk offsets are 32-bit in the kernel.
  return run_len >= 1024 && run_len < (1LL << 31) && n >= (1LL << 20);
}

static int launch_append_runs(const KvAppendParams& p, bool nf, bool cf, DeviceInfo* dev,
                              cudaStream_t st) {
  KvRunParams r;
  r.k_cache = p.k_cache;
  r.v_cache = p.v_cache;
  r.new_k = p.new_k;
  r.new_v = p.new_v;
  const long long slot0 = p.ring ? (long long)p.position % p.slots : p.position;
  const uint64_t row = p.cache_seq_major ? (uint64_t)p.heads * p.head_dim : (uint64_t)p.head_dim;
  r.runs = p.cache_seq_major ? (uint32_t)p.batch : (uint32_t)(p.batch * p.heads);
  r.run_len = (uint32_t)(p.count * row);
  r.chunks_per_run = (r.run_len + kRunChunk - 1) / kRunChunk;
  r.src_run_stride = r.run_len;
  r.dst_run_stride = (uint64_t)p.slots * row;
  r.dst_first = (uint64_t)slot0 * row;
  const int slot = (nf ? 2 : 0) + (cf ? 1 : 0);
  void (*const kern[4])(const KvRunParams) = {
      kv_append_runs_kernel<false, false>, kv_append_runs_kernel<false, true>,
      kv_append_runs_kernel<true, false>, kv_append_runs_kernel<true, true>};
  const uint32_t smem = nf ? run_smem_bytes<true>() : run_smem_bytes<false>();
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!dev->append_runs_ready[slot]) {
      const cudaError_t e =
          cudaFuncSetAttribute(kern[slot], cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return cuda_fail("kv_append smem attribute", e, GQA_ATTN_ERR_LAUNCH);
      dev->append_runs_ready[slot] = true;
    }
  }
  const long long items = 2LL * r.runs * r.chunks_per_run;
  const long long cap = (long long)kRunCtasPerSm * dev->sms;
  const long long blocks = items < cap ? items : cap;
  kern[slot]<<<(unsigned)blocks, kRunThreads, smem, st>>>(r);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? GQA_ATTN_OK : cuda_fail("launch(kv_append runs)", e, GQA_ATTN_ERR_LAUNCH);
}

int gqa_attn_kv_append(void* k_cache, void* v_cache, const void* new_k, const void* new_v,
                       int batch, int cache_slots, int num_kv_heads, int head_dim, int position,
                       int count, unsigned int flags, int* new_length, void* stream) {
  long long n = 0;
  int rc = append_checks(k_cache, v_cache, new_k, new_v, batch, cache_slots, num_kv_heads,
                         head_dim, position, count, flags, &n);
  if (rc != GQA_ATTN_OK) return rc;
  if (new_length) *new_length = position + count;
  if (n == 0) return GQA_ATTN_OK;
  const bool ring = (flags & GQA_KV_RING) != 0;
  DeviceInfo* dev = nullptr;
  rc = device_info(&dev);
  if (rc != GQA_ATTN_OK) return rc;
  KvAppendParams p;
  p.k_cache = k_cache;
  p.v_cache = v_cache;
  p.new_k = new_k;
  p.new_v = new_v;
  p.batch = batch;
  p.heads = num_kv_heads;
  p.slots = cache_slots;
  p.head_dim = head_dim;
  p.position = position;
  p.count = count;
  p.cache_seq_major = (flags & GQA_KV_CACHE_SEQ_MAJOR) ? 1 : 0;
  p.new_head_major = (flags & GQA_KV_NEW_HEAD_MAJOR) ? 1 : 0;
  p.ring = ring ? 1 : 0;
  const long long chunks = 2 * n / 8;  // 8 elements per thread, keys then values
  cudaStream_t st = (cudaStream_t)stream;
  const bool nf = !(flags & GQA_KV_NEW_BF16), cf = (flags & GQA_KV_CACHE_F32) != 0;
  if (append_runs_eligible(p, n)) return launch_append_runs(p, nf, cf, dev, st);
  // One wave: as many blocks as are resident at once (the grid-stride loop
  // takes the rest), so no second partial wave trails the first.
  const int slot = (nf ? 2 : 0) + (cf ? 1 : 0);
  void (*const kern[4])(const KvAppendParams) = {
      kv_append_kernel<false, false>, kv_append_kernel<false, true>,
      kv_append_kernel<true, false>, kv_append_kernel<true, true>};
  int per_sm;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (dev->append_blocks[slot] <= 0) {
      int nb = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kern[slot], 256, 0) != cudaSuccess ||
          nb < 1) {
        (void)cudaGetLastError();
        nb = 1;
      }
      dev->append_blocks[slot] = nb;
    }
    per_sm = dev->append_blocks[slot];
  }
  long long blocks = (chunks + 255) / 256;
  if (blocks > (long long)per_sm * dev->sms) blocks = (long long)per_sm * dev->sms;
  kern[slot]<<<(unsigned)blocks, 256, 0, st>>>(p);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? GQA_ATTN_OK : cuda_fail("launch(kv_append)", e, GQA_ATTN_ERR_LAUNCH);
}

int gqa_attn_decode_append(const void* q, void* k_cache, void* v_cache, const void* new_k,
                           const void* new_v, void* o, int batch, int q_len, int position,
                           int cache_slots, int num_q_heads, int num_kv_heads, int head_dim,
                           unsigned int flags, int causal, int window, float softcap,
                           void* stream) {
  if (flags & GQA_KV_CACHE_F32) return GQA_ATTN_ERR_ARG;  // attention reads bf16 caches
  const bool ring = (flags & GQA_KV_RING) != 0;
  if (position < 0 || cache_slots < 0 ||
      (long long)position + q_len > (ring ? 0x7fffffffLL : (long long)cache_slots))
    return GQA_ATTN_ERR_ARG;
  Problem pr;
  int rc = validate(batch, q_len, position + q_len, num_q_heads, num_kv_heads, head_dim, causal,
                    window, softcap, &pr);
  if (rc != GQA_ATTN_OK) return rc;
  pr.kv_alloc = cache_slots;
  pr.kv_seq_major = (flags & GQA_KV_CACHE_SEQ_MAJOR) ? 1 : 0;
  if (ring && (rc = set_ring(&pr, cache_slots)) != GQA_ATTN_OK) return rc;
  rc = check_pointers(pr, q, k_cache, v_cache, o);
  if (rc != GQA_ATTN_OK) return rc;
  const size_t o_bytes = (size_t)batch * num_q_heads * (size_t)q_len * head_dim * 2;
  const size_t new_bytes = (size_t)batch * num_kv_heads * (size_t)q_len * head_dim *
                           ((flags & GQA_KV_NEW_BF16) ? 2 : 4);
  const size_t q_bytes = o_bytes, cache_bytes = (size_t)batch * num_kv_heads *
                                                  (size_t)cache_slots * head_dim * 2;
  if (overlaps(o, o_bytes, new_k, new_bytes) || overlaps(o, o_bytes, new_v, new_bytes) ||
      overlaps(q, q_bytes, k_cache, cache_bytes) || overlaps(q, q_bytes, v_cache, cache_bytes))
    return GQA_ATTN_ERR_ALIAS;
  long long n_new = 0;
  rc = append_checks(k_cache, v_cache, new_k, new_v, batch, cache_slots, num_kv_heads, head_dim,
                     position, q_len, flags, &n_new);
  if (rc != GQA_ATTN_OK || n_new == 0) return rc;
  DeviceInfo* dev = nullptr;
  if ((rc = device_info(&dev)) != GQA_ATTN_OK) return rc;
  Plan pl;
  if ((rc = make_plan(pr, *dev, &pl)) != GQA_ATTN_OK) return rc;
  if (pl.path == kPathDecode) {
    // One launch: the decode kernel writes the new tokens itself.
    pr.app_count = q_len;
    pr.app_pos = position;
    pr.app_new_f32 = (flags & GQA_KV_NEW_BF16) ? 0 : 1;
    pr.app_new_head_major = (flags & GQA_KV_NEW_HEAD_MAJOR) ? 1 : 0;
    pr.app_new_k = new_k;
    pr.app_new_v = new_v;
    return run(pr, q, k_cache, v_cache, o, (cudaStream_t)stream);
  }
  rc = gqa_attn_kv_append(k_cache, v_cache, new_k, new_v, batch, cache_slots, num_kv_heads,
                          head_dim, position, q_len, flags, nullptr, stream);
  if (rc != GQA_ATTN_OK) return rc;
  return run(pr, q, k_cache, v_cache, o, (cudaStream_t)stream);
}

int gqa_attn_fwd_ring(const void* q, const void* k_ring, const void* v_ring, void* o, int batch,
                      int q_len, int kv_len, int ring_slots, int num_q_heads, int num_kv_heads,
                      int head_dim, unsigned int flags, int causal, int window, float softcap,
                      void* stream) {
  if (flags & ~GQA_KV_CACHE_SEQ_MAJOR) return GQA_ATTN_ERR_ARG;
  Problem pr;
  int rc = validate(batch, q_len, kv_len, num_q_heads, num_kv_heads, head_dim, causal, window,
                    softcap, &pr);
  if (rc != GQA_ATTN_OK) return rc;
  pr.kv_seq_major = (flags & GQA_KV_CACHE_SEQ_MAJOR) ? 1 : 0;
  if ((rc = set_ring(&pr, ring_slots)) != GQA_ATTN_OK) return rc;
  rc = check_pointers(pr, q, k_ring, v_ring, o);
  if (rc != GQA_ATTN_OK) return rc;
  return run(pr, q, k_ring, v_ring, o, (cudaStream_t)stream);
}

const char* gqa_attn_last_error_detail(void) { return g_detail; }

int gqa_attn_fwd_static_scratch(const void* q, const void* k, const void* v, void* o, int batch,
                                int q_len, int kv_len, int num_q_heads, int num_kv_heads,
                                int head_dim, int causal, int window, float softcap,
                                void* stream) {
  Problem pr;
  int rc = validate(batch, q_len, kv_len, num_q_heads, num_kv_heads, head_dim, causal, window,
                    softcap, &pr);
  if (rc != GQA_ATTN_OK) return rc;
  rc = check_pointers(pr, q, k, v, o);
  if (rc != GQA_ATTN_OK) return rc;
  DeviceInfo* dev = nullptr;
  rc = device_info(&dev);
  if (rc != GQA_ATTN_OK) return rc;
  void* scratch = nullptr;
  rc = static_scratch(&scratch);  // first call on a device: symbol lookup
  if (rc != GQA_ATTN_OK) return rc;
  cudaStream_t s = (cudaStream_t)stream;
  if (pr.batch == 0 || pr.q_len == 0) return GQA_ATTN_OK;
  if (pr.kv_len == 0) {
    const size_t bytes = (size_t)pr.batch * pr.hq * (size_t)pr.q_len * pr.d * 2;
    const cudaError_t e = cudaMemsetAsync(o, 0, bytes, s);
    return e == cudaSuccess ? GQA_ATTN_OK : cuda_fail("cudaMemsetAsync(o)", e, GQA_ATTN_ERR_LAUNCH);
  }
  Plan pl;
  rc = plan_decode(pr, *dev, &pl);
  if (rc != GQA_ATTN_OK) return rc;
  if (pl.splits == 1) return launch_decode(pr, pl, *dev, q, k, v, o, nullptr, nullptr, s);
  if (pl.ticket_bytes > kStaticTicketBytes ||
      pl.ws_bytes > kStaticScratchBytes - kStaticTicketBytes) {
    snprintf(g_detail, sizeof g_detail,
             "static scratch too small: needs %zu bytes of partials and %zu of tickets, "
             "has %zu and %zu", pl.ws_bytes, pl.ticket_bytes,
             kStaticScratchBytes - kStaticTicketBytes, kStaticTicketBytes);
    return GQA_ATTN_ERR_TOO_LARGE;
  }
  // Tickets must start at zero; the array keeps whatever the last call left.
  const cudaError_t e = cudaMemsetAsync(scratch, 0, pl.ticket_bytes, s);
  if (e != cudaSuccess) return cuda_fail("cudaMemsetAsync(tickets)", e, GQA_ATTN_ERR_LAUNCH);
  return launch_decode(pr, pl, *dev, q, k, v, o, (char*)scratch + kStaticTicketBytes, scratch, s);
}

}  // extern "C"
