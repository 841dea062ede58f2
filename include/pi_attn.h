/*
 * pi_attn.h -- C ABI of libpiattn.so: the pi0 / pi0.5 joint (prefix-LM)
 * attention on one NVIDIA B200 (sm_100a).
 *
 * What is computed (sources: page title, section):
 *
 *  - "π0.5 vs MM-DiT joint attention", "joint attention 只管算子,mask 才管权限":
 *    each expert's q, k, v are concatenated along the token axis into one
 *    shared KV pool and a single softmax runs over it.  The experts share the
 *    head geometry: 8 query heads, 1 KV head, head_dim 256 (also "Pi0-FAST
 *    模型架构", 6 关键超参数: num_heads 8, num_kv_heads 1, head_dim 256).
 *  - same page, "π0.5:三段,两处看不到": key j is visible to query i iff
 *    cumsum(ar_mask)[j] <= cumsum(ar_mask)[i]; pi0.5 additionally forbids
 *    expert queries from reading FAST keys (last row of the permission table).
 *  - "VLA 代码精读 - OpenPI & StarVLA", 1.2 (Prefix-Suffix 注意力掩码): ar_mask
 *    False = shares attention with the preceding tokens, True = the preceding
 *    tokens cannot see this token.
 *  - same page, 1.6 Pi0.sample_actions: the prefix is run once and its K/V
 *    kept; each of the 10 Euler steps runs only the suffix tokens, whose
 *    queries see every cached prefix key plus the suffix keys allowed by the
 *    cumsum rule over the suffix alone.  The cache is read, never appended.
 *
 *   out[b,i,h,:] = sum_j softmax_j( scale * <q[b,i,h,:], k[b,j,g(h),:]> | visible(i,j) ) v[b,j,g(h),:]
 *   g(h) = h / (Hq / Hkv)
 *
 * Around it (same page, 1.5 and 1.6): pi_rope_inplace rotates q and k at the
 * positions cumsum(mask) - 1 (continued after the prefix in a suffix pass) and
 * pi_euler_update takes the sampler's step x += dt * v.  For training (1.5),
 * pi_attn_prefill_backward returns the gradient of the prefill.
 *
 * Memory layout (all entry points): every tensor is a dense, contiguous,
 * caller-owned DEVICE buffer in token-major order [B, S, H, d] (d innermost,
 * then heads, then tokens, then batch).  ar_mask is uint8 (0 = False,
 * nonzero = True); segment_ids is int32 (PI_SEG_*; a negative value marks a
 * padding token, any other unknown value is treated as PI_SEG_OTHER).  Both
 * are [S] rows, one per batch element at a distance of
 * desc->mask_batch_stride elements (0 = one row shared by the whole batch).
 *
 * Ownership and threading: the library never allocates, frees or retains a
 * caller buffer; all work is enqueued on the caller's stream and the calls
 * return before it runs.  Buffers must stay valid until the stream reaches the
 * work.  Calls on different streams may run concurrently; the global state is
 * the device status word read by pi_attn_read_status, the wait bound set by
 * pi_attn_set_wait_limit, and the fixed scratch of pi_attn_suffix_noalloc.
 * The device addresses of the status word and of that scratch are looked up
 * on every call (cudaGetSymbolAddress, a host-side lookup that is allowed
 * during stream capture), so they stay right after a device reset
 * (cudaDeviceReset) reloads the module; the kernels' shared-memory attributes
 * are set on every call for the same reason; each device's SM count is looked
 * up once and kept.
 *
 * Errors: every entry point returns PI_OK or a PI_ERR_* code.  Argument
 * errors are detected on the host before anything is enqueued (nothing is
 * launched).  PI_ERR_CUDA reports a failed launch (the CUDA error is left in
 * the runtime's sticky/last-error state).  Device-side failures (a bounded
 * wait that ran out) do not trap: the kernel records PI_ERR_TIMEOUT in the
 * status word, abandons its tile and returns, and the host reads it with
 * pi_attn_read_status.  No exception crosses this boundary.
 */
#ifndef PI_ATTN_H_
#define PI_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t (NULL = the legacy default stream), kept opaque here so that
 * C callers need no CUDA headers. */
typedef void* pi_stream_t;

enum pi_dtype {
  PI_BF16 = 0, /* bf16 in/out, fp32 accumulation (tcgen05 tensor cores)   */
  PI_F32 = 1   /* fp32 in/out, fp32 FFMA arithmetic (CUDA cores)         */
};

enum pi_status {
  PI_OK = 0,
  PI_ERR_ARG = 1,         /* NULL pointer, bad shape, stride or size      */
  PI_ERR_ALIGN = 2,       /* a pointer is not 16-byte aligned             */
  PI_ERR_UNSUPPORTED = 3, /* dtype / head geometry the library lacks     */
  PI_ERR_CUDA = 4,        /* a CUDA launch or runtime call failed         */
  PI_ERR_TIMEOUT = 5      /* a device-side bounded wait ran out           */
};

enum pi_segment {
  PI_SEG_PAD = -1,   /* any negative id: a padding token (see below)     */
  PI_SEG_OTHER = 0,  /* prefix: image patches, text, discrete state      */
  PI_SEG_FAST = 1,   /* FAST discrete action tokens                      */
  PI_SEG_EXPERT = 2  /* the action expert's continuous chunk             */
};

/*
 * Padding.  The pages' workloads have none, but openpi ANDs a per-token
 * validity mask (input_mask) into the attention mask ("VLA 代码精读 - OpenPI &
 * StarVLA", 1.5 Pi0.compute_loss; also "Pi0-FAST 模型架构", 2.3).  Here a
 * padding token (negative segment id) is visible to no query and its own
 * query row sees no key.  A query row with no visible key writes out = 0 and
 * lse = -inf.  In the suffix pass, pi_attn_suffix_masked additionally takes a
 * per-batch validity mask for the cached prefix keys.
 */

typedef struct pi_attn_desc {
  int32_t B;    /* batch size (B == 0 is a no-op)                            */
  int32_t Sq;   /* query tokens: prefill = S; suffix = suffix tokens          */
  int32_t P;    /* suffix mode: cached prefix tokens; prefill: must be 0      */
  int32_t Hq;   /* query heads                                                */
  int32_t Hkv;  /* key/value heads; Hq % Hkv == 0                             */
  int32_t d;    /* head dimension                                             */
  int32_t dtype;          /* enum pi_dtype                                    */
  float softmax_scale;    /* multiplies q.k before the softmax (finite, > 0)  */
  int64_t mask_batch_stride; /* elements between batch rows of ar_mask and
                                segment_ids; 0 = shared by the batch, else >= Sq */
} pi_attn_desc;

/*
 * Supported geometry:
 *   PI_BF16: Hkv == 1, d == 256, Hq in {1, 2, 4, 8, 16}; tokens Sq <= 16383
 *            (the in-kernel block index is 14 bits), P < 2^31 / Hq.
 *   PI_F32 : Hq % Hkv == 0, d in {32, 64, 128, 256}, Sq <= 16383.
 * Anything else returns PI_ERR_UNSUPPORTED.  Sq == 0 or B == 0 is a no-op.
 */

/*
 * pi_attn_prefill -- joint prefill over [prefix, suffix] tokens (mode 1).
 * Source: "VLA 代码精读 - OpenPI & StarVLA", 1.5 Pi0.compute_loss (one forward
 * over the concatenated tokens under make_attn_mask), with the mask rule of
 * "π0.5 vs MM-DiT joint attention", π0.5:三段.
 *
 *   q    [B, S, Hq, d]     (S = desc->Sq, desc->P must be 0)
 *   k, v [B, S, Hkv, d]
 *   ar_mask     [B or 1, S] uint8            (required)
 *   segment_ids [B or 1, S] int32 or NULL    (NULL: no expert<-FAST rule, no
 *                                             padding; negative = padding)
 *   out  [B, S, Hq, d]  same dtype as q      (written)
 *   lse  [B, S, Hq] fp32 or NULL             (natural-log log-sum-exp of the
 *                                             scaled visible scores; written)
 * Every non-padding query sees at least itself; a padding row writes 0 and
 * lse = -inf.
 */
int pi_attn_prefill(const pi_attn_desc* desc, const void* q, const void* k, const void* v,
                    const uint8_t* ar_mask, const int32_t* segment_ids, void* out, float* lse,
                    pi_stream_t stream);

/*
 * pi_attn_prefill_ws -- pi_attn_prefill with scratch for a split last round.
 * The bf16 kernel hands whole 256-row query tiles to the SM pairs in rounds;
 * when the last round would leave at least half the pairs idle (MM-DiT: 532
 * tiles on 74 pairs leave 14 for the 8th round), the full rounds run whole
 * and each remaining tile is split over several pairs by key tiles (pieces
 * of at least 6 of the S / 128 key tiles, so short sequences stay whole), its
 * fp32 partials merged by a second kernel (log-sum-exp rule).  Same results
 * up to the rounding order of fp32 sums.
 *   desc ... lse   as pi_attn_prefill
 *   workspace  device scratch of pi_attn_prefill_workspace_bytes(desc) bytes,
 *              16-byte aligned, caller-owned, contents ignored; one call at a
 *              time per workspace.  NULL: as pi_attn_prefill.
 *   ws_bytes   its size
 * Only bf16 with a batch-shared mask (mask_batch_stride == 0) uses it (the
 * size is 0 otherwise).  The size depends on the device's SM count.
 * Errors: as pi_attn_prefill, plus PI_ERR_ARG for a workspace smaller than
 * required and PI_ERR_ALIGN for a misaligned one, before anything is
 * enqueued.
 */
size_t pi_attn_prefill_workspace_bytes(const pi_attn_desc* desc);
/* Pieces per last-round query tile that pi_attn_prefill_ws would split into on
 * the current device (1: no split; the call then launches one kernel, else
 * two).  Host only. */
int pi_attn_prefill_tail_splits(const pi_attn_desc* desc);
int pi_attn_prefill_ws(const pi_attn_desc* desc, const void* q, const void* k, const void* v,
                       const uint8_t* ar_mask, const int32_t* segment_ids, void* out, float* lse,
                       void* workspace, size_t ws_bytes, pi_stream_t stream);

/*
 * pi_attn_prefill_backward -- gradient of pi_attn_prefill with respect to q,
 * k and v, for training.
 * Source: "VLA 代码精读 - OpenPI & StarVLA", 1.5 Pi0.compute_loss runs the
 * joint forward under gradient; the pages print no backward, so this is the
 * plain derivative of the forward: with P the softmax over the visible keys,
 * dS = P * (dO v^T - rowsum(dO * out)), dq = scale dS k, dk = scale dS^T q,
 * dv = P^T dO, the key/value gradients summed over the query heads of each
 * key/value head.
 *
 *   desc        as pi_attn_prefill (P = 0); dtype bf16 or fp32, any Hq that
 *               Hkv divides, d a multiple of 32 up to 256, S <= 16383
 *   q, k, v, ar_mask, segment_ids   the forward's inputs, same layouts
 *   out  [B, S, Hq, d], lse [B, S, Hq] fp32   the forward's outputs (required)
 *   dout [B, S, Hq, d]  same dtype as q       (gradient of the loss w.r.t. out)
 *   dq   [B, S, Hq, d]  fp32                  (written)
 *   dk, dv [B, S, Hkv, d] fp32                (written; not accumulated into)
 *   workspace   device scratch of pi_attn_prefill_backward_workspace_bytes(desc)
 *               bytes, 16-byte aligned, caller-owned, contents ignored
 * Padding tokens (negative segment id) get zero gradients.  The result does not
 * depend on launch timing (no atomics).  Errors: PI_ERR_ARG (bad descriptor,
 * NULL pointer, workspace too small), PI_ERR_ALIGN (a tensor or the workspace
 * not 16-byte aligned, lse / segment_ids not 4-byte aligned),
 * PI_ERR_UNSUPPORTED (geometry above), PI_ERR_CUDA (launch failure); all
 * before anything is enqueued except the last.
 */
size_t pi_attn_prefill_backward_workspace_bytes(const pi_attn_desc* desc);
int pi_attn_prefill_backward(const pi_attn_desc* desc, const void* q, const void* k,
                             const void* v, const uint8_t* ar_mask, const int32_t* segment_ids,
                             const void* out, const float* lse, const void* dout, float* dq,
                             float* dk, float* dv, void* workspace, size_t ws_bytes,
                             pi_stream_t stream);

/*
 * pi_attn_suffix -- suffix-only pass against a prefix KV cache (mode 2), the
 * call each Euler flow-matching step makes.
 * Source: "VLA 代码精读 - OpenPI & StarVLA", 1.6 Pi0.sample_actions: the key
 * mask is [every prefix key | make_attn_mask(suffix ar_mask)], the cache is
 * not extended.
 *
 *   q_suf [B, Sq, Hq, d];  k_suf, v_suf [B, Sq, Hkv, d]
 *   k_cache, v_cache [B, P, Hkv, d]  (read only; P = desc->P >= 0)
 *   ar_mask_suf [B or 1, Sq] uint8
 *   out [B, Sq, Hq, d]
 *   workspace / ws_bytes: caller-provided device scratch of at least
 *   pi_attn_suffix_workspace_bytes(desc) bytes (may be NULL when that is 0);
 *   its contents need no initialisation and are garbage afterwards.  Calls
 *   that may overlap on the GPU need distinct workspaces.
 * Two kernels serve this call.  A suffix of at most 8 query rows (Sq * Hq <=
 * 8, e.g. the single-token decode of "Pi0-FAST 模型架构", 4.1) streams the cache
 * through a cluster of 8 CTAs per batch element (warp-level mma.sync tensor
 * instructions) and merges on chip: it needs no workspace.  Larger suffixes run on the tensor cores;
 * batches too small to fill the GPU split the cache over several CTA pairs
 * and need a workspace for the partial results.
 */
int pi_attn_suffix(const pi_attn_desc* desc, const void* q_suf, const void* k_suf,
                   const void* v_suf, const void* k_cache, const void* v_cache,
                   const uint8_t* ar_mask_suf, void* out, void* workspace, size_t ws_bytes,
                   pi_stream_t stream);

/* Bytes of workspace pi_attn_suffix needs for this descriptor (0 if none);
 * returns 0 for a descriptor that pi_attn_suffix would reject. */
size_t pi_attn_suffix_workspace_bytes(const pi_attn_desc* desc);

/*
 * pi_attn_suffix_masked -- pi_attn_suffix with padding (see "Padding" above).
 *   segment_ids_suf [B or 1, Sq] int32 or NULL: tags of the suffix tokens, at
 *     desc->mask_batch_stride like ar_mask_suf; negative = padding.  The
 *     expert<-FAST rule applies among suffix tokens as in the prefill.
 *   cache_valid [B, P] uint8 or NULL: nonzero = the cached prefix key is valid;
 *     invalid keys are visible to no suffix query.  NULL = every key valid.
 * Everything else (arguments, layout, workspace, errors) as pi_attn_suffix,
 * which is this call with both masks NULL.  segment_ids_suf must be 4-byte
 * aligned (PI_ERR_ALIGN).
 */
int pi_attn_suffix_masked(const pi_attn_desc* desc, const void* q_suf, const void* k_suf,
                          const void* v_suf, const void* k_cache, const void* v_cache,
                          const uint8_t* ar_mask_suf, const int32_t* segment_ids_suf,
                          const uint8_t* cache_valid, void* out, void* workspace,
                          size_t ws_bytes, pi_stream_t stream);

/*
 * pi_attn_debug_mask -- writes the visibility matrix the kernels evaluate, as
 * uint8 0/1, for bit-exact comparison with an explicitly built mask.
 * Uses the same in-kernel predicate (cumsum of ar_mask, the expert<-FAST
 * rule, and the suffix-pass prefix columns) as the attention kernels.
 *   mode 0 (prefill): mask_out [B, Sq, Sq];      seg may be NULL (negative = padding)
 *   mode 1 (suffix) : mask_out [B, Sq, P + Sq];  seg must be NULL (no cache mask)
 * Only desc->B, Sq, P and mask_batch_stride are read.
 */
int pi_attn_debug_mask(const pi_attn_desc* desc, int mode, const uint8_t* ar_mask,
                       const int32_t* segment_ids, uint8_t* mask_out, pi_stream_t stream);

/*
 * pi_attn_debug_tiles -- writes the tile classes the bf16 prefill kernel uses
 * to skip work, for comparison with a brute-force scan of the explicit mask.
 * The kernel walks 256-row query tiles (256 / Hq tokens x Hq heads) against
 * 128-key tiles; for each pair it decides from the block indices, the FAST /
 * expert tags and the padding flags of the tokens (the rule of "π0.5 vs
 * MM-DiT joint attention", π0.5:三段,两处看不到) that no row sees any key
 * (skipped), that every row sees every key (full) or neither (partial, masked
 * per element).  This call runs the same scan and classification.
 *   desc         B, Sq (= S), Hq and mask_batch_stride are read; P must be 0;
 *                Hq in {1, 2, 4, 8, 16}
 *   ar_mask, segment_ids   as pi_attn_prefill (device memory)
 *   classes_out  device uint8 [B][ceil(S*Hq/256)][ceil(S/128)]: 0 skipped,
 *                1 full, 2 partial
 * Errors: PI_ERR_ARG, PI_ERR_ALIGN, PI_ERR_UNSUPPORTED before any launch;
 * PI_ERR_CUDA if the launch fails.
 */
int pi_attn_debug_tiles(const pi_attn_desc* desc, const uint8_t* ar_mask,
                        const int32_t* segment_ids, uint8_t* classes_out, pi_stream_t stream);

/*
 * pi_attn_read_status -- synchronises `stream`, returns the device status word
 * (PI_OK or the first PI_ERR_TIMEOUT recorded by any kernel since the last
 * read) and clears it.  Returns PI_ERR_CUDA if the synchronisation fails.
 */
int pi_attn_read_status(pi_stream_t stream);

/* Human-readable name of a pi_status code (static storage). */
const char* pi_attn_status_string(int status);

/*
 * pi_attn_set_wait_limit -- bound, in SM clock cycles, on every device-side
 * spin wait (mbarrier phase waits) in kernels launched after this call.
 * 0 restores the default (2^31 cycles, about a second).  Returns the previous
 * value.  Process-wide.  The value in force when the library is loaded is the
 * environment variable PIATTN_WATCHDOG_CYCLES (a positive decimal integer)
 * if set, else the default.
 *
 * Every entry point that enqueues work opens an NVTX range named after itself
 * for its host-side duration (inert unless a profiler is attached).
 */
uint64_t pi_attn_set_wait_limit(uint64_t cycles);

/*
 * pi_attn_selftest_wait -- launches one CTA that waits on an mbarrier that
 * nothing ever arrives at, bounded by the current wait limit; the wait runs
 * out and records PI_ERR_TIMEOUT in the status word.  Exercises the timeout
 * path of the same bounded-wait routine the attention kernels use, without
 * faulting or hanging the GPU.
 */
int pi_attn_selftest_wait(pi_stream_t stream);

/*
 * pi_attn_suffix_noalloc -- pi_attn_suffix for callers that cannot allocate
 * device memory.  The pages have no counterpart: this is plumbing, not part of
 * the method.  Same arguments, layout, result and errors as pi_attn_suffix,
 * minus the workspace: the split-K partials go to a fixed buffer inside the
 * library (a file-scope __device__ array, one per device, of
 * pi_attn_suffix_noalloc_capacity() = 16 MiB).
 *
 *  - Allocates nothing: no cudaMalloc/cudaFree, no allocating library call.
 *  - Each call looks up the buffer's address (cudaGetSymbolAddress) on the
 *    current device; the lookup also works during stream capture.
 *  - Nothing in the buffer needs to start at zero: every call writes each
 *    partial it later reads.
 *  - Two calls that may overlap on the GPU (different streams of one device)
 *    race on the shared buffer and give wrong results; calls on one stream are
 *    ordered and safe.  Different devices have separate buffers.
 *  - PI_ERR_UNSUPPORTED, before anything is enqueued, when the descriptor
 *    needs more than the capacity (pi_attn_suffix_workspace_bytes(desc) >
 *    16 MiB; that happens only for small-batch shapes with many query rows).
 */
int pi_attn_suffix_noalloc(const pi_attn_desc* desc, const void* q_suf, const void* k_suf,
                           const void* v_suf, const void* k_cache, const void* v_cache,
                           const uint8_t* ar_mask_suf, void* out, pi_stream_t stream);

/* Size in bytes of the fixed buffer pi_attn_suffix_noalloc uses. */
size_t pi_attn_suffix_noalloc_capacity(void);

/*
 * Steps on either side of the attention (the Euler sampling loop of
 * "VLA 代码精读 - OpenPI & StarVLA", 1.6 Pi0.sample_actions).
 *
 * pi_rope_inplace -- rotary position embedding of q (and k) in place.
 * Positions are cumsum(token_mask) - 1 over the call's S tokens (1.5: the
 * joint forward), and with a prefix mask they continue after its valid
 * tokens: sum(prefix_mask) + cumsum(token_mask) - 1 (1.6: the suffix pass).
 * The pages name the LLM's built-in RoPE without a formula; this is the
 * standard rotation of each head vector's (i, i + d/2) pairs by the angle
 * pos * base^(-2i/d):  [x1 cos - x2 sin, x2 cos + x1 sin].
 *   q [B, S, Hq, d], k [B, S, Hkv, d] or NULL  (bf16 or fp32, rotated in place)
 *   token_mask [B or 1, S] uint8 (nonzero = valid token), at mask_batch_stride
 *   prefix_mask [B or 1, P] uint8 at prefix_batch_stride; required iff P > 0
 *   positions_out [B, S] int32 or NULL (written: the positions used)
 * d must be a multiple of 16 and at most 256, B at most 65535, and one
 * token's heads, (Hq + Hkv) * d * element size (Hkv counted only when k is
 * given), at most 160 KiB (else PI_ERR_UNSUPPORTED); base > 1 (10000 for
 * Gemma).  The kernel has no device-side waits.
 * Errors as the attention calls (host-side checks, PI_ERR_ALIGN for pointers
 * not 16-byte aligned).
 */
typedef struct pi_rope_desc {
  int32_t B, S, P;         /* batch, tokens to rotate, prefix tokens (0 = none) */
  int32_t Hq, Hkv, d;      /* heads of q and k, head dimension                   */
  int32_t dtype;           /* PI_BF16 or PI_F32 (q and k alike)                  */
  float base;              /* rotary base, > 1                                   */
  int64_t mask_batch_stride;    /* token_mask: 0 = shared by the batch, else >= S */
  int64_t prefix_batch_stride;  /* prefix_mask: 0 = shared, else >= P             */
} pi_rope_desc;

int pi_rope_inplace(const pi_rope_desc* desc, void* q, void* k, const uint8_t* token_mask,
                    const uint8_t* prefix_mask, int32_t* positions_out, pi_stream_t stream);

/*
 * pi_euler_update -- one Euler step of the flow-matching sampler in place,
 * x <- x + dt * v (1.6: dt = -1 / num_steps, from t = 1 to t = 0).
 *   x [n] fp32 (the action chunk, read and written), v [n] bf16 or fp32
 *   (v_dtype PI_BF16 / PI_F32).  Both 16-byte aligned.
 */
int pi_euler_update(float* x, const void* v, int32_t v_dtype, float dt, int64_t n,
                    pi_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* PI_ATTN_H_ */
