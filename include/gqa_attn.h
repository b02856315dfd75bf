/*
 * gqa_attn.h -- C ABI of libgqa_attn.so: masked grouped-query attention
 * forward pass on NVIDIA B200 (sm_100a).
 *
 * Operation ("TPU v6e Masked GQA Kernel Optimization", sections "What You
 * Have" and "What You Submit"): for bf16 q (batch, num_q_heads, q_len,
 * head_dim) and k, v (batch, num_kv_heads, kv_len, head_dim) return
 *
 *     o = softmax(mask(softcap(q . k^T / sqrt(head_dim)))) . v
 *
 * as bf16 with q's shape, for GQA ratios num_q_heads / num_kv_heads >= 1
 * (the pages' family is 1:1 to 16:1), with an optional causal mask, an
 * optional sliding window and an optional logit softcap s * tanh(x / s).
 * The arguments mirror the cfg dict of that page's make_attention(cfg)
 * entry point (its "seed" and "name" fields are harness-only and not
 * passed).
 *
 * Conventions (the pages are silent on them; these are the readings used by
 * both the CUDA path and the test oracle):
 *   - layout: every tensor is dense, row-major, contiguous, bf16, device
 *     memory: q and o are [batch][num_q_heads][q_len][head_dim], k and v are
 *     [batch][num_kv_heads][kv_len][head_dim].
 *   - q head h reads kv head h / (num_q_heads / num_kv_heads) (contiguous
 *     groups, the same as repeat-interleaving the kv heads).
 *   - query i sits at position qpos = kv_len - q_len + i (bottom-right
 *     alignment of both masks).
 *   - key j is visible iff j < kv_len
 *         && (!causal     || j <= qpos)
 *         && (window <= 0 || (0 <= qpos - j && qpos - j < window)).
 *     A window of W therefore sees W keys ending at qpos, and implies j <= qpos
 *     even without `causal`.
 *   - logits: x = (q . k) / sqrt(head_dim) with the logical head_dim; if
 *     softcap > 0 then x = softcap * tanh(x / softcap); masking follows.
 *   - softmax in fp32 over the visible keys (the pages' baseline uses an fp32
 *     softmax); P is rounded to bf16 for the P.V product on the tensor cores;
 *     o is rounded to bf16 (round to nearest even).
 *   - a row with no visible key returns zeros (never NaN).
 *   - results are deterministic: the same inputs on the same device give
 *     bitwise the same output ("Deterministic: same inputs, same output",
 *     section "Hard Constraints").
 *
 * Accuracy target: |o - ref| <= 2e-2 + 2e-2 * |ref| elementwise against an
 * fp32-or-better reference ("How It Is Judged": rtol=2e-2, atol=2e-2).
 */
#ifndef GQA_ATTN_H
#define GQA_ATTN_H

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes (negative = the call did nothing). */
#define GQA_ATTN_OK 0
#define GQA_ATTN_ERR_NULL_POINTER (-1) /* a tensor with elements has a NULL pointer */
#define GQA_ATTN_ERR_MISALIGNED (-2)   /* a pointer is not 16-byte aligned */
#define GQA_ATTN_ERR_BAD_SHAPE (-3)    /* a negative size, zero heads, or int overflow */
#define GQA_ATTN_ERR_HEAD_RATIO (-4)   /* num_q_heads % num_kv_heads != 0 */
#define GQA_ATTN_ERR_HEAD_DIM (-5)     /* head_dim not a multiple of 8 in [8, 256] */
#define GQA_ATTN_ERR_SOFTCAP (-6)      /* softcap negative, NaN or infinite */
#define GQA_ATTN_ERR_DEVICE (-7)       /* current device is not compute capability 10.x */
#define GQA_ATTN_ERR_LAUNCH (-8)       /* a CUDA launch or copy failed */
#define GQA_ATTN_ERR_ALLOC (-9)        /* workspace allocation failed */
#define GQA_ATTN_ERR_TOO_LARGE (-10)   /* a dimension exceeds what the kernels index */
#define GQA_ATTN_ERR_ALIAS (-11)       /* o overlaps q, k or v */
#define GQA_ATTN_ERR_ARG (-12)         /* another invalid argument */

/* Bits of the sticky device status word (gqa_attn_status). */
#define GQA_ATTN_STATUS_TIMEOUT_LOADER 0x1u
#define GQA_ATTN_STATUS_TIMEOUT_COMPUTE 0x2u
#define GQA_ATTN_STATUS_TIMEOUT_MMA 0x4u
#define GQA_ATTN_STATUS_TIMEOUT_SOFTMAX 0x8u
#define GQA_ATTN_STATUS_TIMEOUT_EPILOGUE 0x10u
#define GQA_ATTN_STATUS_TIMEOUT_SELFTEST 0x20u

/*
 * gqa_attn_fwd -- o = masked GQA attention(q, k, v).
 *
 * q, k, v: device pointers (read only), o: device pointer (written), layouts
 * above, 16-byte aligned; o must not overlap q, k or v.  The caller owns all
 * four buffers and the stream; pointers may be NULL only for tensors with no
 * elements.  Sizes: batch, q_len, kv_len >= 0; num_q_heads, num_kv_heads >= 1
 * with num_q_heads % num_kv_heads == 0; head_dim % 8 == 0, 8 <= head_dim <=
 * 256.  causal: 0 or non-zero.  window <= 0 means no window.  softcap == 0
 * means no softcap; otherwise finite and > 0.  stream: a cudaStream_t (NULL =
 * the legacy default stream) on the current device.
 *
 * The call validates, plans and enqueues 1 kernel (a memset when kv_len == 0,
 * nothing when o is empty) on `stream` and returns without synchronising.
 * Key-split partials live in a library-owned workspace per (device, stream),
 * allocated with cudaMalloc on first need; calls on one stream are ordered,
 * calls on different streams do not share workspace.  A call that needs more
 * than the stream's workspace allocates a bigger one (no synchronisation)
 * and retires the old one without freeing it, so a CUDA graph captured
 * earlier on that stream keeps valid pointers; gqa_attn_release_workspace
 * frees everything.  Partials of the split-KV decode kernel and of the
 * tcgen05 kernel's key splits use the workspace.  The last CTA of a unit to
 * finish merges them, except when every (batch, kv head) has one 128-row
 * tile split into 2 to 8 CTAs and all of the grid's CTAs fit on the device
 * at once: then the tcgen05 kernel is launched as one thread-block cluster
 * per (batch, kv head), whose CTAs meet at the cluster barrier and merge a
 * column slice each (gqa_attn_describe_merge tells which).
 *
 * CUDA graphs: a call of a given size on a stream enqueues only kernels (and
 * allocates nothing) once a call of that size has run on that stream, so
 * capture after one direct call.
 *
 * Returns GQA_ATTN_OK or a negative GQA_ATTN_ERR_* code.  Errors raised while
 * the kernel runs surface at the next synchronisation (CUDA convention) and,
 * for bounded-wait timeouts, in gqa_attn_status().
 */
int gqa_attn_fwd(const void* q, const void* k, const void* v, void* o, int batch, int q_len,
                 int kv_len, int num_q_heads, int num_kv_heads, int head_dim, int causal,
                 int window, float softcap, void* stream);

/*
 * gqa_attn_fwd_host -- the same computation for inputs and output in host
 * memory.  q_host, k_host, v_host (read) and o_host (written) are host
 * pointers, best page-locked (cudaHostAlloc) so the copies are asynchronous.
 * q_dev, k_dev, v_dev, o_dev are caller-owned device buffers of the same
 * sizes (16-byte aligned).  Enqueues on `stream`: three host-to-device copies,
 * the attention kernel, one device-to-host copy -- one cudaMemcpyAsync per
 * tensor -- then waits for the stream.  Returns as gqa_attn_fwd.
 */
int gqa_attn_fwd_host(const void* q_host, const void* k_host, const void* v_host, void* o_host,
                      void* q_dev, void* k_dev, void* v_dev, void* o_dev, int batch, int q_len,
                      int kv_len, int num_q_heads, int num_kv_heads, int head_dim, int causal,
                      int window, float softcap, void* stream);

/*
 * gqa_attn_describe -- the plan gqa_attn_fwd would use for these sizes on
 * the current device, without launching anything.  Any output pointer may
 * be NULL.  *path: 0 = nothing to do, 1 = split-KV decode kernel, 2 = tcgen05
 * prefill kernel, 3 = zero fill (kv_len == 0).  *splits: key chunks per row
 * block (decode) or key-range splits per row tile (tcgen05 kernel; 1 = none).
 * *ctas: work items of the launch (CTAs, or items of the persistent grid).
 * *tiles: key tiles of the widest row block.  Returns GQA_ATTN_OK or the error gqa_attn_fwd would
 * return for these sizes.
 */
int gqa_attn_describe(int batch, int q_len, int kv_len, int num_q_heads, int num_kv_heads,
                      int head_dim, int causal, int window, float softcap, int* path, int* splits,
                      int* ctas, int* tiles);

/*
 * gqa_attn_set_override -- test and tuning knobs (process-wide).
 * key 1: force the path (value 0 = automatic, 1 = decode, 2 = prefill);
 * key 2: force the number of key tiles per decode split (0 = automatic);
 * key 3: force the number of key splits of the tcgen05 kernel for units with
 *        one row tile (rounded up to even; 0 = automatic);
 * key 4: how those splits merge (0 = automatic: by every CTA of one
 *        thread-block cluster per unit when a unit has 2 to 8 CTAs and the
 *        whole grid fits on the device at once; -1 = always by the last CTA
 *        of a unit to finish);
 * key 5: 1 = the tcgen05 kernel's softcap path always finds the row max
 *        before the exponentials (0 = automatic: caps up to about 63.8 use a
 *        fixed exponent base and a single pass over the scores).
 * A forced path that cannot run these sizes falls back to automatic.
 * Returns GQA_ATTN_OK or GQA_ATTN_ERR_ARG for an unknown key.
 */
int gqa_attn_set_override(int key, int value);

/* Human-readable text for a GQA_ATTN_* return code (static storage). */
const char* gqa_attn_error_string(int status);

/*
 * gqa_attn_describe_merge -- how gqa_attn_fwd would merge key-split partials
 * for these sizes on the current device: *cluster = CTAs per thread-block
 * cluster of the distributed-shared-memory merge, or 0 (workspace merge, or
 * no splits).  Launches nothing.  Returns as gqa_attn_describe.
 */
int gqa_attn_describe_merge(int batch, int q_len, int kv_len, int num_q_heads, int num_kv_heads,
                            int head_dim, int causal, int window, float softcap, int* cluster);

/*
 * gqa_attn_status -- the sticky device status word of the current device
 * (GQA_ATTN_STATUS_* bits, 0 = nothing happened), read with a synchronous
 * copy; call after synchronising.  Returns -1 when it cannot be read.
 *
 * gqa_attn_clear_status resets it to 0 and zeroes the split-ticket counters
 * of every workspace of the current device: a kernel that gave up a bounded
 * wait may have left a count behind, which would make a later split merge
 * run early or never.  Call it after synchronising, with no call of this
 * library in flight on the device, before using the device again after a
 * non-zero status; it synchronises the device.  Returns GQA_ATTN_OK or an
 * error.
 */
int gqa_attn_status(void);
int gqa_attn_clear_status(void);

/*
 * gqa_attn_release_workspace -- synchronise every device that holds a
 * workspace of this library and free all of them (active and retired).
 * Graphs captured before must not be replayed afterwards; the next call
 * allocates afresh.  Returns GQA_ATTN_OK or GQA_ATTN_ERR_LAUNCH.
 */
int gqa_attn_release_workspace(void);

/*
 * gqa_attn_selftest_bounded_wait -- failure-detection self test: launches
 * one CTA that waits on an mbarrier nothing will complete, with a wait limit
 * of `limit_us` microseconds (1..10,000,000).  The kernel gives up, sets
 * GQA_ATTN_STATUS_TIMEOUT_SELFTEST and returns; no trap, the context stays
 * usable.  Enqueued on `stream`; returns GQA_ATTN_OK or an error code.
 */
int gqa_attn_selftest_bounded_wait(int limit_us, void* stream);

/*
 * gqa_attn_last_error_detail -- for the calling thread, which CUDA call
 * failed last and its error name ("" when none); static thread-local
 * storage, overwritten by the next failure.
 */
const char* gqa_attn_last_error_detail(void);

/*
 * gqa_attn_fwd_static_scratch -- gqa_attn_fwd for callers that cannot
 * allocate device memory, restricted to the split-KV decode kernel.
 *
 * The pages describe no such entry point; it exists for callers who may not
 * call cudaMalloc: code whose device memory is all handed to its own pool
 * (an allocation outside the pool fails or fragments it), and latency-bound
 * callers that cannot take the device-wide synchronisation cudaMalloc and
 * cudaFree can cause.  gqa_attn_fwd allocates its split workspace on first
 * need; this variant allocates nothing and calls no allocating routine.
 *
 * Arguments, layouts, ownership and return codes are those of gqa_attn_fwd;
 * the computation is always the split-KV decode kernel (any sizes it takes,
 * head_dim up to 256).  Its scratch (split partials and tickets) is one
 * file-scope device array of 8 MiB (64 KiB of tickets + 8128 KiB of
 * partials) that every GPU loading this library holds until the process
 * exits.  A plan whose partials or tickets exceed it returns
 * GQA_ATTN_ERR_TOO_LARGE (see gqa_attn_last_error_detail); plans with one
 * split use no scratch.  Each call clears the tickets it uses with
 * cudaMemsetAsync on `stream` before the kernel.
 *
 * The first call on a device looks the array's device address up
 * (cudaGetSymbolAddress, with that device current); make that first call
 * before any stream capture.  All calls share the one array: calls whose
 * execution overlaps on the GPU (other streams, other threads) race on it,
 * so serialise them.
 */
int gqa_attn_fwd_static_scratch(const void* q, const void* k, const void* v, void* o, int batch,
                                int q_len, int kv_len, int num_q_heads, int num_kv_heads,
                                int head_dim, int causal, int window, float softcap,
                                void* stream);

/* ---------------------------------------------------------- KV cache append
 * Flags for gqa_attn_kv_append and gqa_attn_decode_append (bitwise or). */
#define GQA_KV_CACHE_SEQ_MAJOR 0x1u /* caches [batch][slots][kv_heads][d]; else [batch][kv_heads][slots][d] */
#define GQA_KV_CACHE_F32 0x2u       /* caches hold fp32; else bf16 */
#define GQA_KV_NEW_BF16 0x4u        /* new keys/values are bf16; else fp32 */
#define GQA_KV_NEW_HEAD_MAJOR 0x8u  /* new keys/values [batch][kv_heads][count][d]; else [batch][count][kv_heads][d] */
#define GQA_KV_RING 0x10u           /* ring cache: token p goes to slot p % cache_slots (see below) */

/*
 * Write the keys and values of `count` new tokens into a key cache and a
 * value cache at slots [position, position + count) ("KV Cache Update at a
 * Position", TensorTonic, problem statement and constraints): in every batch
 * row and kv head, slot position + l receives new token l, converted to the
 * cache dtype (fp32 -> bf16 rounds to nearest even; bf16 -> fp32 is exact);
 * every other slot keeps its contents.  *new_length (a host int; may be
 * NULL) receives position + count, the page's returned `length`.
 *
 * Layouts (dense, row-major, device memory, 16-byte aligned): the caches are
 * [batch][cache_slots][num_kv_heads][head_dim] with GQA_KV_CACHE_SEQ_MAJOR
 * (the page's layout) and [batch][num_kv_heads][cache_slots][head_dim]
 * without it (the layout gqa_attn_fwd reads); the new keys and values are
 * [batch][count][num_kv_heads][head_dim] (the page's) or, with
 * GQA_KV_NEW_HEAD_MAJOR, [batch][num_kv_heads][count][head_dim].  The caller
 * owns every buffer; the call allocates nothing and is asynchronous on
 * `stream` (a cudaStream_t; NULL = legacy default stream).
 *
 * With GQA_KV_RING the caches are rings (the layouts above with cache_slots
 * slots): token position + l goes to slot (position + l) % cache_slots, so
 * position may exceed cache_slots; count must not (the block would
 * overwrite itself).
 *
 * Errors (nothing is launched): GQA_ATTN_ERR_ARG for unknown flags or
 * position < 0 or position + count > cache_slots (ring: count > cache_slots
 * or position + count > INT_MAX); GQA_ATTN_ERR_BAD_SHAPE,
 * GQA_ATTN_ERR_HEAD_DIM, GQA_ATTN_ERR_NULL_POINTER, GQA_ATTN_ERR_MISALIGNED
 * as for gqa_attn_fwd; GQA_ATTN_ERR_ALIAS if the two caches overlap or a new
 * buffer overlaps a cache.  count == 0 (or batch == 0) launches nothing.
 */
int gqa_attn_kv_append(void* k_cache, void* v_cache, const void* new_k, const void* new_v,
                       int batch, int cache_slots, int num_kv_heads, int head_dim, int position,
                       int count, unsigned int flags, int* new_length, void* stream);

/*
 * One decode step on a KV cache: append the q_len new tokens' keys and
 * values at `position` (gqa_attn_kv_append with the same flags), then
 * attend q -- the same q_len tokens -- to cache slots [0, position + q_len)
 * exactly as gqa_attn_fwd with kv_len = position + q_len, so query i sits at
 * position + i.  Both steps run in order on `stream`; the attention reads
 * the caches in place, in either layout, with no copy.
 *
 * With GQA_KV_RING the caches are rings and the attention is that of
 * gqa_attn_fwd_ring with kv_len = position + q_len and ring_slots =
 * cache_slots.
 *
 * The caches must be bf16 (GQA_KV_CACHE_F32 returns GQA_ATTN_ERR_ARG).  q
 * and o are [batch][num_q_heads][q_len][head_dim] bf16.  Return codes are
 * those of both calls; GQA_ATTN_ERR_ALIAS also when q overlaps a cache or o
 * overlaps a cache, q or a new buffer.  The output equals, bit for bit,
 * gqa_attn_fwd on contiguous copies of the caches' first position + q_len
 * slots.
 */
int gqa_attn_decode_append(const void* q, void* k_cache, void* v_cache, const void* new_k,
                           const void* new_v, void* o, int batch, int q_len, int position,
                           int cache_slots, int num_q_heads, int num_kv_heads, int head_dim,
                           unsigned int flags, int causal, int window, float softcap,
                           void* stream);

/*
 * Masked GQA attention over keys and values kept in ring buffers (decode
 * over a sliding window stored circularly): key j of the kv_len-key
 * sequence lives in slot j % ring_slots of k_ring / v_ring, which are
 * [batch][num_kv_heads][ring_slots][head_dim] bf16, or
 * [batch][ring_slots][num_kv_heads][head_dim] with GQA_KV_CACHE_SEQ_MAJOR
 * (the only flag accepted).  The result is that of gqa_attn_fwd on the keys
 * in order -- same mask rule, query i at kv_len - q_len + i -- provided the
 * ring still holds every key a query can see: ring_slots >= min(kv_len,
 * q_len + window - 1) with a window, ring_slots >= kv_len without one.  So a
 * ring of window + q_len - 1 slots serves a sliding window of `window`.
 * (Decode rows over ring windows: "CSA2 attention on Metal", TensorFold
 * pull request 1709, section "What this changes".)
 *
 * ring_slots must be a positive multiple of 64.  Computed by the split-KV
 * decode kernel whatever the number of rows.  Errors: those of
 * gqa_attn_fwd, and GQA_ATTN_ERR_ARG for a bad ring_slots, a ring too small
 * for the visible keys (see gqa_attn_last_error_detail) or unknown flags.
 */
int gqa_attn_fwd_ring(const void* q, const void* k_ring, const void* v_ring, void* o, int batch,
                      int q_len, int kv_len, int ring_slots, int num_q_heads, int num_kv_heads,
                      int head_dim, unsigned int flags, int causal, int window, float softcap,
                      void* stream);

/* Library version as major * 10000 + minor * 100 + patch. */
int gqa_attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GQA_ATTN_H */
