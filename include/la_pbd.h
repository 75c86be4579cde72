/*
 * la_pbd.h -- C ABI of the B200 (sm_100a) Parallel Box Decoding window-attention library.
 *
 * What the library computes
 * -------------------------
 * One PBD decode step of LocateAnything-3B attends a window of W query tokens (the last
 * accepted token plus 5 <text_mask> tokens, so W = 6; W = 1 is plain next-token decoding)
 * over the decoder's KV cache. Inside the window attention is bidirectional; toward the
 * prefix it is causal, so every window row sees cache rows [0, P_b + W) of its sequence and
 * nothing beyond (LocateAnything-3B for RK3588 model card, "How it differs from the
 * original", item 1). The decoder is Qwen2.5-3B: 36 layers, K/V tensors of shape
 * [1, 2, seq, 128] per layer (LocateAnything-3B ONNX WebGPU INT4 model card, "KV-cache graph
 * for in-browser use"), hidden size 2048 (same card, "Why this repo exists"), so 16 query
 * heads share 2 KV heads; bf16 throughout ("LocateAnything-3B on a 12 GB RTX 4000 Ada",
 * "Architecture footprint").
 *
 * For sequence b, query head h, window row i (position P_b + i):
 *   s_j  = scale * <q[b,i,h,:], k[b, h / (Hq/Hkv), j, :]>          j in [0, P_b + W)
 *   out[b,i,h,:] = sum_j softmax_j(s) * v[b, h / (Hq/Hkv), j, :]
 * computed with bf16 inputs, fp32 accumulation, bf16 (round-to-nearest-even) output.
 *
 * Layouts (all row-major, contiguous, device memory unless stated)
 *   q, out         bf16 [B, W, Hq, D]
 *   k_cache,v_cache bf16 [B, Hkv, S_max, D]   one row = D * 2 = 256 bytes, 16-byte aligned
 *   k_new, v_new   bf16 [B, W, Hkv, D]       window keys/values, RoPE already applied
 *   seq_lens       int32 [B]                 committed prefix length P_b of each sequence
 *
 * Ownership: the caller owns every buffer. The compute entry points never allocate, free or
 * synchronise; they enqueue work on `stream` (a cudaStream_t passed as void*; NULL = legacy
 * default stream) and return. They are reentrant. Run la_kv_append before la_pbd_attn on the
 * same stream (or use la_pbd_step, which does both).
 *
 * Stream order: the kernels are launched with programmatic dependent launch, so each may
 * start before the previous kernel of the stream has finished; each waits for it
 * (griddepcontrol.wait) before reading anything a predecessor may have written, so stream
 * order holds as usual. A caller's own kernel launched after one of these calls with
 * programmatic dependent launch must, as that mechanism requires of any kernel, write
 * nothing that the call reads (seq_lens, window_lens, the block table, q, the caches)
 * before its own griddepcontrol.wait.
 *
 * Errors: static arguments are checked on the host and reported synchronously (nothing is
 * enqueued on error). Per-sequence errors found on the device (seq_lens[b] < 0 or
 * seq_lens[b] + W > max_seq) never fault: that sequence's output rows are written as zeros,
 * its cache is left untouched, and a sticky flag is raised in the workspace header, read and
 * cleared by la_pbd_check. Kernel launch failures map to LA_ERR_CUDA.
 */
#ifndef LA_PBD_H_
#define LA_PBD_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum la_status {
  LA_OK = 0,
  LA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misaligned pointer               */
  LA_ERR_UNSUPPORTED = 2,   /* head_dim != 128, Hq % Hkv != 0, W * Hq/Hkv too large ... */
  LA_ERR_WORKSPACE = 3,     /* workspace missing or smaller than la_pbd_workspace_bytes */
  LA_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed                        */
  LA_ERR_SEQ_OVERFLOW = 5,  /* (la_pbd_check) a sequence had P < 0 or P + W > max_seq   */
  LA_ERR_TIMEOUT = 6        /* (la_pbd_check) a bounded device-side wait gave up        */
} la_status;

/* Mask applied inside the window. */
enum {
  LA_MASK_PBD = 0,            /* bidirectional inside the window (the trained model)       */
  LA_MASK_CAUSAL_WINDOW = 1   /* causal inside the window: row i sees [0, P_b + i]; the
                                 RKLLM approximation (RK3588 card, item 1)                 */
};

/* Kernel selection. */
enum {
  LA_ALGO_AUTO = 0,      /* tensor-core kernel when supported, else CUDA cores             */
  LA_ALGO_TCGEN05 = 1,   /* tcgen05 (TMEM accumulators) + TMA staging; W * Hq/Hkv <= 80    */
  LA_ALGO_SIMT = 2       /* fp32 CUDA-core kernel; W * Hq/Hkv <= 128                       */
};

typedef struct la_pbd_cfg {
  int32_t batch;         /* B >= 1, B <= 4096                                              */
  int32_t num_q_heads;   /* Hq, a multiple of num_kv_heads                                  */
  int32_t num_kv_heads;  /* Hkv >= 1                                                        */
  int32_t head_dim;      /* D; must be 128                                                  */
  int32_t max_seq;       /* S_max, cache rows per (sequence, KV head); B*Hkv*S_max < 2^31   */
  float scale;           /* softmax scale, usually 1/sqrt(D)                                */
  int32_t mask_mode;     /* LA_MASK_*                                                       */
  int32_t algo;          /* LA_ALGO_*                                                       */
} la_pbd_cfg;

/* Library version as 10000*major + 100*minor + patch. */
int32_t la_version(void);

/* Static text for a status code (never NULL). */
const char* la_status_string(la_status status);

/*
 * The attention kernel that la_pbd_attn / la_pbd_step / la_pbd_attn_varwin would run for this
 * configuration and (longest) window length: LA_ALGO_TCGEN05 or LA_ALGO_SIMT. With
 * cfg->algo = LA_ALGO_AUTO the choice follows the measured per-workload timing of both kernels
 * on B200 (the tensor-core kernel wherever it supports the shape, W * Hq/Hkv <= 80). Host
 * only; returns -la_status for an invalid or unsupported configuration.
 */
int32_t la_pbd_algo(const la_pbd_cfg* cfg, int32_t window_len);

/*
 * Bytes of device workspace la_pbd_attn / la_pbd_step need for this configuration and window
 * length on the current device: a 256-byte header (sticky error flags) followed by the
 * per-split partial results (running max, running sum, unnormalised fp32 output rows), which
 * a second (merge) kernel of the same call combines.
 * Returns 0 if the configuration is invalid or unsupported.
 */
size_t la_pbd_workspace_bytes(const la_pbd_cfg* cfg, int32_t window_len);

/*
 * Zero the workspace header (error flags) on `stream`. Call once after allocating a workspace;
 * the partial-result area needs no initialisation.
 */
la_status la_pbd_workspace_init(void* workspace, size_t workspace_bytes, void* stream);

/*
 * Step a1 -- window K/V append (RK3588 card, item 1: the prefix KV is reused, the window's
 * tokens are written after it, with no rollback of stale speculative rows).
 * For every b, w < W, KV head h:  k_cache[b, h, P_b + w, :] = k_new[b, w, h, :]  (same for v).
 * Bit-exact copy. Sequences with P_b < 0 or P_b + W > max_seq are skipped (la_pbd_attn then
 * flags them). k_new/v_new must not alias the caches.
 */
la_status la_kv_append(const la_pbd_cfg* cfg, const void* k_new, const void* v_new,
                       void* k_cache, void* v_cache, const int32_t* seq_lens,
                       int32_t window_len, void* stream);

/*
 * Steps a2..a6 -- PBD window attention over the cache (window rows already appended).
 * q, out: bf16 [B, W, Hq, D]; caches bf16 [B, Hkv, S_max, D]; seq_lens int32 [B] on the
 * device; 1 <= window_len <= 16. `workspace` must hold la_pbd_workspace_bytes(cfg, W) bytes
 * whose header was zeroed once by la_pbd_workspace_init. out may not alias any input.
 */
la_status la_pbd_attn(const la_pbd_cfg* cfg, const void* q, const void* k_cache,
                      const void* v_cache, const int32_t* seq_lens, int32_t window_len,
                      void* out, void* workspace, size_t workspace_bytes, void* stream);

/*
 * One whole layer call: the result of la_kv_append followed by la_pbd_attn on the same
 * stream (same caches afterwards, same output bits). With the tcgen05 kernel (LA_ALGO_AUTO
 * with W * Hq/Hkv <= 80, or LA_ALGO_TCGEN05) both run in one launch: the attention kernel
 * reads the window's keys and values from k_new / v_new and writes them into the caches
 * itself (the fused append; RK3588 model card, "How it differs from the original", item 1:
 * the window's rows are placed after the reused prefix, with no rollback). k_new and v_new
 * must not alias the caches. Validation, errors and the treatment of invalid prefix lengths
 * (no cache write, zero output rows, sticky flag) are those of the two calls.
 */
la_status la_pbd_step(const la_pbd_cfg* cfg, const void* q, const void* k_new,
                      const void* v_new, void* k_cache, void* v_cache,
                      const int32_t* seq_lens, int32_t window_len, void* out,
                      void* workspace, size_t workspace_bytes, void* stream);

/*
 * la_pbd_attn without a caller-provided workspace, for callers that cannot allocate device
 * memory: a plugin inside a host engine that owns all device memory and offers its kernels no
 * scratch, or a latency-critical loop in which cudaMalloc is not allowed because it can
 * synchronise the device and take an unbounded time. The paper has no counterpart; this is a
 * deployment convenience of this library.
 * Runs the same kernels as la_pbd_attn with their scratch in one file-scope device array of
 * 32 MiB that every GPU loading the library holds until the process exits; the call itself
 * allocates and frees nothing. Configurations whose la_pbd_workspace_bytes exceeds 32 MiB are
 * rejected with LA_ERR_WORKSPACE (nothing enqueued); a valid configuration that cannot be
 * sized because a device query failed gives LA_ERR_CUDA. Every call looks up the array's device
 * address (cudaGetSymbolAddress) with the current device. Under CUDA's lazy module loading (the
 * default since CUDA 12.2) the first call on each device loads the library's code there and
 * reserves the array, which may allocate and synchronise: make that first call during set-up,
 * outside any latency-critical loop, and before any stream capture. All calls on a device share
 * the one array and it keeps the last call's contents: calls whose executions overlap on the
 * GPU (other streams, concurrent threads) race on it and must be serialised by the caller.
 * Nothing in it needs to start at zero (every value a kernel reads was written earlier in the
 * same call). Device-side per-sequence errors still produce zero rows, but their sticky flag
 * stays in the shared array and is not readable through la_pbd_check.
 */
la_status la_pbd_attn_static(const la_pbd_cfg* cfg, const void* q, const void* k_cache,
                             const void* v_cache, const int32_t* seq_lens, int32_t window_len,
                             void* out, void* stream);

/*
 * Window attention with a window length per sequence (the RKLLM engine's step sends each
 * sequence's accepted tokens plus 5 <text_mask> tokens, so W_b differs within a batch: RK3588
 * model card, "How it differs from the original", item 1). Same as la_pbd_attn with W =
 * W_max for the layouts, except:
 *   window_lens  device int32 [B], 1 <= W_b <= W_max
 *   q, out       bf16 [B, W_max, Hq, D]: rows i < W_b of sequence b are its window (row i
 *                at position P_b + i, seeing keys [0, P_b + W_b), or [0, P_b + i] with
 *                LA_MASK_CAUSAL_WINDOW); rows i >= W_b are padding, never read into the
 *                result, and written as zeros.
 * A sequence with P_b < 0, W_b outside [1, W_max] or P_b + W_b > max_seq gets zero rows and
 * raises the sticky flag (la_pbd_check). workspace: la_pbd_workspace_bytes(cfg, W_max).
 */
la_status la_pbd_attn_varwin(const la_pbd_cfg* cfg, const void* q, const void* k_cache,
                             const void* v_cache, const int32_t* seq_lens,
                             const int32_t* window_lens, int32_t window_max, void* out,
                             void* workspace, size_t workspace_bytes, void* stream);

/*
 * One layer call with per-sequence windows: rows w < W_b of k_new / v_new (bf16
 * [B, W_max, Hkv, D]) are appended at cache rows P_b + w (padding rows are not), then
 * la_pbd_attn_varwin. Fused into one launch with the tcgen05 kernel, as in la_pbd_step.
 */
la_status la_pbd_step_varwin(const la_pbd_cfg* cfg, const void* q, const void* k_new,
                             const void* v_new, void* k_cache, void* v_cache,
                             const int32_t* seq_lens, const int32_t* window_lens,
                             int32_t window_max, void* out, void* workspace,
                             size_t workspace_bytes, void* stream);

/*
 * Paged KV cache (tcgen05 kernel only, i.e. W * Hq/Hkv <= 80 and algo != LA_ALGO_SIMT, else
 * LA_ERR_UNSUPPORTED). The caches are page pools
 *   k_pool, v_pool  bf16 [num_pages, Hkv, page_size, D]
 *   block_table     device int32 [B, pages_per_seq]: key j of sequence b lives in page
 *                   block_table[b][j / page_size], row j % page_size
 * page_size a multiple of 64 (each 128-key tile is read as 64-row boxes). A sequence holds
 * at most pages_per_seq * page_size keys (this replaces cfg->max_seq for the capacity check);
 * the table entries of pages [0, ceil((P_b + W) / page_size)) must be valid pages, later
 * entries are never read. Otherwise as la_pbd_attn / la_pbd_step (the step appends the window
 * rows into their pages, fused into the attention launch).
 */
la_status la_pbd_attn_paged(const la_pbd_cfg* cfg, const void* q, const void* k_pool,
                            const void* v_pool, const int32_t* block_table,
                            int32_t pages_per_seq, int32_t page_size, int32_t num_pages,
                            const int32_t* seq_lens, int32_t window_len, void* out,
                            void* workspace, size_t workspace_bytes, void* stream);
la_status la_pbd_step_paged(const la_pbd_cfg* cfg, const void* q, const void* k_new,
                            const void* v_new, void* k_pool, void* v_pool,
                            const int32_t* block_table, int32_t pages_per_seq,
                            int32_t page_size, int32_t num_pages, const int32_t* seq_lens,
                            int32_t window_len, void* out, void* workspace,
                            size_t workspace_bytes, void* stream);

/*
 * Bytes of device workspace la_block_prefill needs for this configuration and t_max: the
 * 256-byte header, one int32 per 128-row V tile and an fp16 copy of V
 * (B * Hkv * ceil(t_max / 128) * 128 rows of D channels, 256 bytes each). Host only.
 * Returns 0 for an invalid configuration or t_max < 1.
 */
size_t la_block_prefill_workspace_bytes(const la_pbd_cfg* cfg, int32_t t_max);

/*
 * Block-causal prefill attention (the block mask of block-diffusion decoding over whole
 * sequences; the PBD window is the last block of it): token i of sequence b attends key j
 * when j <= i or when both lie in the same block of block_size consecutive tokens, i.e. j <
 * min(T_b, (i / block_size + 1) * block_size).
 *   q, out         bf16 [B, t_max, Hq, D] (rows i >= T_b of out are written as zeros)
 *   k_cache,v_cache bf16 [B, Hkv, S_max, D] with the sequence's keys/values in rows [0, T_b)
 *   seq_lens       device int32 [B]: T_b, 0 <= T_b <= min(t_max, S_max)
 *   block_size     >= 1
 *   workspace      >= la_block_prefill_workspace_bytes(cfg, t_max), 256-byte aligned (its
 *                  header, zeroed by la_pbd_workspace_init, receives the sticky flags read by
 *                  la_pbd_check; the rest needs no initialisation)
 * bf16 inputs, fp32 accumulation, bf16 out. The probabilities enter the PV product in fp16
 * (8x finer than bf16), with V converted to fp16 in the workspace first (exact for
 * 2^-17 <= |v| <= 65504). Where a 128-row V tile that a query tile reads holds a |v| of
 * 65520 or more, or only values below 2^-6 in magnitude, that query tile uses bf16 V with
 * the probabilities as two bf16 parts (P_hi + P_lo) instead. Either way the product keeps
 * fp32-level accuracy in P.
 * A sequence with T_b outside [0, min(t_max, S_max)] gets zero rows and the sticky flag.
 * Asynchronous on `stream` (two kernels: the V conversion, then the attention); allocates
 * nothing.
 */
la_status la_block_prefill(const la_pbd_cfg* cfg, const void* q, const void* k_cache,
                           const void* v_cache, const int32_t* seq_lens, int32_t t_max,
                           int32_t block_size, void* out, void* workspace,
                           size_t workspace_bytes, void* stream);

/*
 * Host-side view of the split-KV work plan that la_pbd_attn follows on the device, for
 * inspection and testing; touches no GPU. The keys [0, P_b + W) of each (sequence b, KV
 * head h) are cut into tiles of `unit_keys` keys (the attention kernel's key tile), and
 * (b, h) occupies `seg_units` units standing for the fixed cost of a segment followed by one
 * unit per tile. All units are laid end to end, and CTA c of `num_ctas` takes one
 * contiguous run of them; the tiles of a (b, h) in one CTA are a segment (a CTA whose run
 * holds only fixed-cost units of (b, h) gets none of it). The attention kernels use
 * unit_keys = 128, seg_units = 3 (tcgen05 kernel) and unit_keys = 32, seg_units = 0
 * (CUDA-core kernel); the tcgen05 kernel uses seg_units = 0 when B * Hkv * ceil(S_max / 128)
 * does not exceed its grid (148 CTAs on B200), where every CTA gets at most one tile.
 * Sequences with an invalid prefix length contribute nothing.
 *   seq_lens_host  host int32 [cfg->batch]
 *   segments       host int32 [max_segments][6], written in CTA order as
 *                  {cta, b, h, j0, j1, slot}: keys [j0, j1) of (b, h); slot = -1 when the
 *                  segment is the whole sequence (its CTA writes the output), else the
 *                  workspace slot of its partial result
 * Returns the number of segments (which may exceed max_segments; only the first
 * max_segments are written), or -la_status on invalid arguments (num_ctas < 1,
 * unit_keys < 1, seg_units < 0, a null pointer, an invalid cfg).
 */
int32_t la_pbd_plan(const la_pbd_cfg* cfg, int32_t window_len, const int32_t* seq_lens_host,
                    int32_t num_ctas, int32_t unit_keys, int32_t seg_units, int32_t* segments,
                    int32_t max_segments);

/*
 * Measurement aid, not part of the attention path (the pages have no counterpart): the
 * benchmark's launch-floor reference. Enqueues `launches` empty kernels of `ctas` x `threads` on `stream`,
 * chained with programmatic dependent launch like the library's own kernels. Timing a CUDA
 * graph of these beside a graph of real calls with the same launch count gives the part of
 * the step that launching alone costs. Asynchronous; allocates nothing. LA_ERR_INVALID_ARG
 * for launches < 0, ctas < 1 or threads outside [1, 1024]; LA_ERR_CUDA if a launch fails.
 */
la_status la_noop_chain(int32_t launches, int32_t ctas, int32_t threads, void* stream);

/*
 * The plan parameters that an attention kernel uses: its key tile (`*unit_keys`) and the
 * fixed segment cost in tiles (`*seg_units`; applied only when a CTA can get several
 * tiles, see la_pbd_plan), for algo LA_ALGO_TCGEN05 or LA_ALGO_SIMT.
 * Host only. LA_ERR_INVALID_ARG for another algo or a null pointer.
 */
la_status la_pbd_plan_params(int32_t algo, int32_t* unit_keys, int32_t* seg_units);

/*
 * Self-test of the device-side failure detection (the pages have no counterpart). Every wait
 * of the tensor-core kernels is bounded: when one runs out, the CTA raises the sticky
 * LA_ERR_TIMEOUT flag in the workspace header, the kernel's other roles stop at their next
 * wait, copies and tensor-core products in flight are drained with bounded waits, tensor
 * memory is freed and the kernel returns, so the context stays usable. This call enqueues one
 * la_pbd_attn on the tcgen05 kernel (the configuration must select it) in which every wait
 * gives up after `wait_limit_ns` (1000 .. 2e9 ns) and the MMA thread withholds the completion
 * signal of its first S^T product, so that the softmax warps' wait for it runs out. The call's
 * `out` is then undefined; la_pbd_check afterwards returns LA_ERR_TIMEOUT and clears it, and
 * the workspace serves the next call as usual. Arguments and errors otherwise as la_pbd_attn.
 */
la_status la_pbd_selftest_timeout(const la_pbd_cfg* cfg, const void* q, const void* k_cache,
                                  const void* v_cache, const int32_t* seq_lens,
                                  int32_t window_len, void* out, void* workspace,
                                  size_t workspace_bytes, int64_t wait_limit_ns, void* stream);

/*
 * The same self-test for the block-causal prefill kernel: one la_block_prefill in which every
 * wait gives up after `wait_limit_ns` (1000 .. 2e9 ns) and the QK^T-issuing thread withholds
 * the completion signal of the first S product of key half 0, so that the wait of that
 * half's softmax warps runs out. The call's `out` is then undefined; la_pbd_check on the
 * workspace afterwards returns LA_ERR_TIMEOUT and clears it, and the workspace serves the
 * next call as usual. Arguments and errors otherwise as la_block_prefill.
 */
la_status la_block_prefill_selftest_timeout(const la_pbd_cfg* cfg, const void* q,
                                            const void* k_cache, const void* v_cache,
                                            const int32_t* seq_lens, int32_t t_max,
                                            int32_t block_size, void* out, void* workspace,
                                            size_t workspace_bytes, int64_t wait_limit_ns,
                                            void* stream);

/*
 * Self-test of the tensor-core kernel's early start (the pages have no counterpart). Before
 * its dependency wait the kernel makes its split plan from seq_lens as they are then; right
 * after the wait it issues the copies of its first segment and makes the plan again from the
 * values after the wait; if the two differ, it drains those copies, initialises its barriers
 * again and follows the new plan. This call enqueues one call in which the comparison is
 * forced to fail, so that the second path runs: la_pbd_attn (k_new and v_new NULL) or
 * la_pbd_step (both given), with the same arguments and results (the same output bits and
 * caches as the normal call). The configuration must select the tcgen05 kernel.
 */
la_status la_pbd_selftest_replan(const la_pbd_cfg* cfg, const void* q, const void* k_new,
                                 const void* v_new, void* k_cache, void* v_cache,
                                 const int32_t* seq_lens, int32_t window_len, void* out,
                                 void* workspace, size_t workspace_bytes, void* stream);

/*
 * Synchronise `stream`, read and clear the workspace's sticky device-side error flags.
 * Returns LA_OK, LA_ERR_SEQ_OVERFLOW, LA_ERR_TIMEOUT or LA_ERR_CUDA.
 */
la_status la_pbd_check(void* workspace, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LA_PBD_H_ */
