/*
 * mk.h -- C ABI of the persistent decode megakernel for B200 (sm_100a).
 *
 * One decode step of a Llama-style dense decoder (RMSNorm + QKV + RoPE, GQA
 * attention over a paged bf16 KV cache, O-projection + residual, RMSNorm +
 * SwiGLU gate/up, down-projection + residual, final norm + LM head + greedy
 * argmax) runs as ONE persistent kernel launch: every SM walks its own
 * precomputed instruction tape, instructions wait on global-memory counters
 * instead of kernel boundaries, and shared memory is a ring of pages into which
 * the next instructions' weights are streamed while the current one computes.
 *
 * Sources of the method: the Hazy Research megakernel article "Stanford team's
 * new work lets Llama-1B reach millisecond inference" (m.youleyou.com/wenzhang/
 * 2897217), section "Megakernel: a deep-fusion design from scratch": one kernel
 * for the whole forward; an on-GPU instruction interpreter; a per-SM execution
 * plan of fused instructions (RMSNorm+QKV+RoPE, attention, MLP); dependencies
 * resolved before the run; paged shared memory so the next stage preloads its
 * weights; completion counters in global memory (atomic +1, waiters spin until
 * a preset value) instead of global barriers.  The interface below is this
 * library's own; the pages define none.
 *
 * Conventions
 *  - All weights are caller-owned DEVICE pointers to bf16, row-major [out, in],
 *    and must stay valid (and unmodified) for the life of the handle.
 *  - Output buffers are caller-owned; the library owns the KV cache, the
 *    scratch activations, the counters and the tapes.
 *  - Calls return an mk_status and never abort the process.  Kernel launches
 *    are asynchronous on the given stream; device-side failures (a bounded wait
 *    that ran out, an out-of-range token) are recorded in a device error word
 *    and reported by mk_sync / mk_get_error.  After such a failure every later
 *    step returns at once until mk_clear_error is called.
 *  - One step at a time per handle: steps of one handle must be ordered on one
 *    stream (or otherwise serialised); two handles may run concurrently.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 */
#ifndef MK_H
#define MK_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct mk_ctx* mk_handle;

typedef enum {
  MK_OK = 0,
  MK_ERR_INVALID_ARG = 1,   /* a NULL pointer, a size or index out of range */
  MK_ERR_UNSUPPORTED = 2,   /* a shape this build does not handle (see mk_create) */
  MK_ERR_OOM = 3,           /* device allocation failed */
  MK_ERR_CUDA = 4,          /* a CUDA runtime call failed (no device, launch error) */
  MK_ERR_TIMEOUT = 5,       /* a bounded wait inside the kernel ran out */
  MK_ERR_DEVICE_FAULT = 6,  /* the kernel reported bad input (e.g. token >= vocab) */
  MK_ERR_ABORTED = 7        /* an earlier device error is pending; see mk_clear_error */
} mk_status;

/* Model shape and capacity.  Requirements checked by mk_create:
 *   head_dim in {64, 128}; n_heads % n_kv_heads == 0 with n_heads/n_kv_heads
 *   in {1, 2, 4, 8}; hidden, ffn multiples of 8; hidden <= 4096 and
 *   n_heads*head_dim <= 8192 (two rows of Wq/Wgate, one row of Wo, fit a
 *   16 KiB page);
 *   1 <= max_batch <= 8; B * max(hidden, n_heads*head_dim) <= 16384 where B is
 *   max_batch rounded up to 1, 2, 4 or 8.
 * RoPE rotates half-split pairs (i, i + head_dim/2) by pos * inv_freq[i],
 * inv_freq[i] = rope_theta^(-2i/head_dim); with rope_scaling != 0 the Llama-3
 * rule (rope_factor, rope_low_freq, rope_high_freq, rope_orig_max) rescales
 * long wavelengths. */
typedef struct {
  int32_t n_layers;
  int32_t hidden;
  int32_t n_heads;
  int32_t n_kv_heads;
  int32_t head_dim;
  int32_t ffn;
  int32_t vocab;
  int32_t tied;            /* 1: LM head is the embedding matrix */
  float rms_eps;
  float rope_theta;
  int32_t rope_scaling;    /* 0: none, 1: Llama-3 frequency scaling */
  float rope_factor;
  float rope_low_freq;
  float rope_high_freq;
  int32_t rope_orig_max;
  int32_t max_batch;       /* sequence slots 0..max_batch-1 */
  int32_t max_seq;         /* positions 0..max_seq-1 per slot */
  int32_t kv_dtype;        /* KV cache element: 0 = bf16, 1 = fp16 (both 2 bytes; fp16
                              keeps 3 more mantissa bits for deep models) */
} mk_config;

/* Device pointers (bf16).  The per-layer members are HOST arrays of n_layers
 * device pointers; mk_create copies them. */
typedef struct {
  const void* embed;        /* [vocab, hidden] */
  const void* lm_head;      /* [vocab, hidden]; NULL iff tied */
  const void* final_norm;   /* [hidden] */
  const void* const* attn_norm;  /* [hidden] each */
  const void* const* wq;         /* [n_heads*head_dim, hidden] */
  const void* const* wk;         /* [n_kv_heads*head_dim, hidden] */
  const void* const* wv;         /* [n_kv_heads*head_dim, hidden] */
  const void* const* wo;         /* [hidden, n_heads*head_dim] */
  const void* const* mlp_norm;   /* [hidden] */
  const void* const* w_gate;     /* [ffn, hidden] */
  const void* const* w_up;       /* [ffn, hidden] */
  const void* const* w_down;     /* [hidden, ffn] */
} mk_weights;

/* Optional knobs (pass NULL for defaults). */
typedef struct {
  int32_t device;            /* CUDA device ordinal (default 0) */
  int32_t wait_limit_ms;     /* bound of every in-kernel wait (default 1000) */
  int32_t n_sm;              /* SMs to use (0 = all) */
  int32_t ring_pages;        /* shared-memory pages in the weight ring (0 = as many as fit) */
  int32_t debug_fault;       /* test hook, 0 in normal use.  1: raise the wait target of
                                one instruction by one, so that wait can never be met and
                                runs out after wait_limit_ms (the step then reports
                                MK_ERR_TIMEOUT and the context stays usable) */
  int32_t profile;           /* 1: every step records per-instruction timestamps
                                (see mk_profile_read); costs a few stores per instruction */
  int32_t dyn_percent;       /* share of the gate/up, down and LM-head rows that SMs claim
                                at run time instead of taking from a fixed range: 0 = none
                                (default), 1..90 = that percent; else MK_ERR_INVALID_ARG */
  int32_t prefill_tokenwise; /* 1: mk_prefill runs every prompt token through the decode
                                kernel, one step per token; 0 (default): prompts of 17 or
                                more tokens run batched on the tensor cores (see mk_prefill) */
  int32_t region_cut;        /* 1: every decode step is two launches of the persistent
                                kernel, the decoder layers and then the final norm + LM head
                                + argmax (the region cut of "One Megakernel is Not Enough:
                                Predicting Where to Cut for Streaming Inference", section
                                "Four observations"); results are identical.  0 (default):
                                one launch per step, or per n steps with mk_decode_steps */
  int32_t tensor_core_units; /* which matvecs of the 8-lane kernel (5-8 lanes) run on the
                                tcgen05 tensor cores (128-row blocks, accumulators in tensor
                                memory) where the shape allows it (the Llama-3.2-1B-shaped
                                kernel): 0 (default) the choice measured faster -- the LM head
                                and gate/up on tcgen05 --, 1 none (CUDA cores everywhere), 2 the
                                LM head, 3 gate/up, 4 both; other values: MK_ERR_INVALID_ARG */
} mk_options;

/* Create a handle: validates the config, lowers it into per-SM instruction
 * tapes (one set per active batch size 1..max_batch), allocates the KV cache
 * (bf16, pages of 16 KiB per layer and kv head) and scratch, zeroes them, and
 * copies the QKV, gate/up and down matrices into device buffers of its own in
 * the order the kernel streams them (each 16 KiB page one contiguous block; the
 * handle then holds a second copy of those matrices, e.g. 1.8 GB for the
 * Llama-3.2-1B shape).
 * Returns MK_ERR_INVALID_ARG / MK_ERR_UNSUPPORTED before touching the GPU when
 * the config or pointers are bad. */
mk_status mk_create(const mk_config* cfg, const mk_weights* w, const mk_options* opt,
                    mk_handle* out);

/* Run one decode step for lanes b = 0..nb-1, lane b using sequence slot b.
 *   tokens_dev    device int32[nb]: the input token of each lane (may be the
 *                 previous step's ids_dev, so steps chain without a host sync)
 *   positions     HOST int32[nb]: absolute position of that token; slot b's
 *                 cache must hold positions 0..pos-1
 *   logits_dev    device float[nb, vocab] or NULL (not written)
 *   ids_dev       device int32[nb]: greedy argmax, lowest index on ties
 * Writes K/V of each lane's position into its slot.  Asynchronous. */
mk_status mk_decode_step(mk_handle h, int32_t nb, const int32_t* tokens_dev,
                         const int32_t* positions, float* logits_dev, int32_t* ids_dev,
                         void* stream);

/* n_steps greedy decode steps in ONE launch, lanes b = 0..nb-1 in slots b.
 * Step 0 reads tokens_dev[b] at positions[b]; step t > 0 reads the id step t-1
 * produced, at positions[b] + t.  ids_dev (device int32[n_steps][nb]) receives
 * every step's ids; logits_dev is NULL or device float[n_steps][nb][vocab].
 * Requires positions[b] + n_steps <= max_seq.  Asynchronous.  The kernel keeps
 * streaming weights across step boundaries, so this is faster per step than
 * n_steps calls of mk_decode_step. */
mk_status mk_decode_steps(mk_handle h, int32_t nb, int32_t n_steps, const int32_t* tokens_dev,
                          const int32_t* positions, float* logits_dev, int32_t* ids_dev,
                          void* stream);

/* The same step with HOST buffers: copies tokens in, runs the step, copies ids
 * (and logits when logits_host != NULL, float[nb, vocab]) back, and waits for
 * the stream.  Returns the step's device status. */
mk_status mk_decode_step_host(mk_handle h, int32_t nb, const int32_t* tokens_host,
                              const int32_t* positions, float* logits_host,
                              int32_t* ids_host, void* stream);

/* Prefill sequence slot `seq` with n HOST tokens at positions start_pos ..
 * start_pos+n-1 (the cache must hold positions 0 .. start_pos-1).  When the shape
 * allows it (hidden, n_heads*head_dim and n_kv_heads*head_dim multiples of 128,
 * ffn a multiple of 64) and n >= 17, tokens 0 .. n-2 run batched, in passes of
 * at most 2048 tokens: per layer RMSNorm, the QKV GEMM on tcgen05 tensor cores
 * (RoPE and the K/V cache writes fused), causal attention over the cache, the O
 * GEMM, the gate/up GEMM (SwiGLU fused) and the down GEMM, with activations split
 * into bf16 high and low parts so the products keep fp32-level accuracy; then the
 * last token runs through the decode kernel.  Otherwise (or with
 * mk_options.prefill_tokenwise) one launch runs one decode step per token.
 * Prefill has the shape of a GEMM where decode has that of a matvec: "One
 * Megakernel is Not Enough: Predicting Where to Cut for Streaming Inference",
 * section "Why where to cut matters more than whether to fuse".
 * logits_last_dev (device float[vocab], nullable) and id_last_host (host int32*,
 * nullable) receive the last position's logits and greedy id; when id_last_host
 * is non-NULL the call waits for the stream.  The prompt is copied before the
 * call returns. */
mk_status mk_prefill(mk_handle h, int32_t seq, const int32_t* tokens_host, int32_t n,
                     int32_t start_pos, float* logits_last_dev, int32_t* id_last_host,
                     void* stream);

/* Wait for `stream` and return the device status of the steps run so far. */
mk_status mk_sync(mk_handle h, void* stream);

/* Decode the device error word into `buf` (always NUL-terminated); returns the
 * status it maps to.  Synchronises the device. */
mk_status mk_get_error(mk_handle h, char* buf, int32_t len);

/* Clear a recorded device error, the abort flag and all counters. */
mk_status mk_clear_error(mk_handle h);

/* Profile records of the last step (handle created with mk_options.profile = 1).
 * Layout: int64 out[n_sm][stride][32]; record i of SM s describes the i-th
 * instruction of that SM's tape: [0] op | layer << 8 | n_units << 24,
 * [1] consumer start, [2] dependency met, [3] units done, [4] counter signalled,
 * [5] producer issued the first unit's page, [6] producer issued the last
 * unit's page (all %globaltimer ns, 0 where not reached); accumulated since the
 * last read: [7] ns the consumer warps waited for their matvec pages,
 * [8] pages they took, [9] ns the producer waited for free ring slots, [10] matvec
 * pages it issued; matvec instructions also record [11] activations staged,
 * [12] the CTA's last warp finished its units, [13] the CTA passed its end
 * barrier (the counter release follows), and accumulate [14] ns the first
 * consumer warps spent in page dot products, [15] ns in the reductions and
 * epilogues, [16] group re-reads of activations not yet written when first
 * loaded, [17] ns those re-reads took (lane 0 of each warp), [18] staging
 * entered, [19] the first staged values back, [20..21] the residual
 * accumulator back (QKV, LM head), [22] the first warp entered its pages,
 * [24] its first page landed; [23], [25..31] unused.  The end stamps [4], [12],
 * [13] are the last warp's (no barrier is added for them).
 * Reading resets the accumulators.
 * `cap` is the capacity of `out` in int64 elements; *n_sm and *stride are set
 * even when out is NULL, so a first call can size the buffer.  Synchronises
 * the device. */
mk_status mk_profile_read(mk_handle h, int64_t* out, int64_t cap, int32_t* n_sm, int32_t* stride);

/* Free everything the library owns (never the caller's weights or outputs). */
mk_status mk_destroy(mk_handle h);

/* ---- host-only introspection (no GPU needed) ---- */

typedef struct {
  int32_t n_instr_total;     /* instructions over all SMs */
  int32_t n_counters;        /* counters per set */
  int32_t max_instr_per_sm;
  int64_t bytes_min_sm;      /* weight + estimated KV bytes streamed per SM */
  int64_t bytes_max_sm;
  int32_t deadlock_free;     /* 1 if the tape simulator ran every instruction */
  int32_t coverage_ok;       /* 1 if every output tile is produced exactly once */
  int32_t targets_ok;        /* 1 if every wait target equals its counter's signal count */
  int32_t attn_slices;       /* attention slices per (lane, kv head) */
  int32_t ring_pages;        /* pages the kernel would use for this shape */
  int32_t smem_bytes;        /* dynamic shared memory per CTA */
} mk_plan_report;

/* Lower `cfg` for `n_sm` SMs and `nb` active lanes, run the CPU tape simulator
 * over the result and fill `rep`.  `dyn_percent` is mk_options.dyn_percent (the
 * share of the streaming phases claimed at run time, 0..90); `region` is the part
 * of the step the tape holds: 0 the whole step, 1 the decoder layers, 2 the final
 * norm + LM head (the two launches of mk_options.region_cut); `tensor_core_units` is
 * mk_options.tensor_core_units (which 8-lane matvecs are tensor-core units).  `fault` != 0 plants
 * a fault in the tape first (1: one signal dropped, 2: one wait target raised by
 * one, 3: one instruction's claim range of the LM head shortened by one row
 * block, with dyn_percent > 0) so tests can see the simulator report it. */
mk_status mk_plan_check(const mk_config* cfg, int32_t n_sm, int32_t nb, int32_t fault,
                        int32_t dyn_percent, int32_t region, int32_t tensor_core_units,
                        mk_plan_report* rep);

/* The RoPE inverse frequencies this library builds its (cos, sin) table from:
 * out[i] = rope_theta^(-2i/head_dim) for i < head_dim/2, rescaled by the Llama-3
 * rule when cfg->rope_scaling != 0 (see mk_config).  Host only, no GPU; the table
 * itself holds cos and sin of pos * out[i], computed in double and rounded to
 * float.  The RoPE rotation is the fused "RMSNorm + QKV + RoPE" instruction of
 * the Hazy megakernel article (section "Megakernel: a deep-fusion design from
 * scratch"); the frequency rule is the published Llama-3 one, which the pages
 * name ("RoPE theta 500000 with Llama-3 scaling") without spelling out.
 *   out  host double[n], n >= head_dim/2 (else MK_ERR_INVALID_ARG) */
mk_status mk_rope_inv_freq(const mk_config* cfg, double* out, int32_t n);

/* ---- greedy head without allocation ----
 *
 * No counterpart in the pages: a convenience entry point of this library.
 *
 * The last stage of a decode step as a stand-alone call on the current CUDA
 * device: for lanes b < nb,
 *   logits[b][v] = lm_head[v] . (x_b / sqrt(mean(x_b^2) + rms_eps) * final_norm)
 *   ids[b]       = argmax_v logits[b][v], lowest index on ties,
 * from a caller-provided hidden state.  It is for callers that run the decoder
 * layers themselves and cannot allocate device memory on their call path: code
 * inside a framework whose caching allocator already owns the GPU's memory, where
 * a raw cudaMalloc can fail or make the whole device wait, and latency-critical
 * loops that allow no allocation once started.  It calls no cudaMalloc/cudaFree.
 *
 * Its only working memory (the per-block argmax partials and a completion
 * counter) is one static device array of MK_NOALLOC_SCRATCH_BYTES, held on every
 * GPU that loads the library until the process exits.  Every call shares it and
 * it keeps the last call's contents; the kernel returns its counter to zero
 * itself.  Calls that overlap on the GPU (e.g. on two streams) race on it: order
 * them on one stream.  The first call on a device looks up the array's device
 * address with that device current; make that first call before any stream
 * capture.  That look-up is kept for the life of the process and is not redone
 * after a cudaDeviceReset, so the entry point is not usable on a device that has
 * been reset.  A call made while an earlier CUDA error is pending on the calling
 * thread returns MK_ERR_CUDA without launching and leaves that error in place.
 *
 *   hidden_dev   device float[nb][hidden]
 *   final_norm   device bf16[hidden];   lm_head  device bf16[vocab][hidden] (16-byte aligned)
 *   logits_dev   device float[nb][vocab] or NULL;   ids_dev  device int32[nb]
 * Limits: 1 <= nb <= 8 and nb * hidden <= 16384 -- larger requests return
 * MK_ERR_UNSUPPORTED without launching; hidden must be a multiple of 8.
 * Asynchronous on `stream`. */
#define MK_NOALLOC_SCRATCH_BYTES 65536
mk_status mk_greedy_head_noalloc(const float* hidden_dev, int32_t nb, int32_t hidden,
                                 const void* final_norm, const void* lm_head, int32_t vocab,
                                 float rms_eps, float* logits_dev, int32_t* ids_dev, void* stream);

/* The two engines a decode step's matvecs can run on, measured apart.
 *
 * The Hazy megakernel article (section "Megakernel: a deep-fusion design from
 * scratch") says tensor cores win again on Blackwell.  This call runs the
 * streaming batched matvec the decode kernel is made of,
 *     Y[b][r] = sum_k W[r][k] * X[b][k],  b < nb,  r < rows,
 * on one engine, so the claim can be checked per batch size:
 *   engine 0  CUDA cores (packed FP32 FMA over bulk-copied pages of whole rows;
 *             the decode kernel's engine); requires K == 2048, rows % 4 == 0;
 *   engine 1  tcgen05 tensor cores: TMA tiles of 128 rows x 64, MMA M = 128,
 *             N = 16 with X split into bf16 high and low parts (fp32-level
 *             accuracy), fp32 accumulators in tensor memory; requires K % 64 == 0,
 *             K <= 4096, rows % 128 == 0.
 *   W  device bf16 [rows][K] row-major, 16-byte aligned (caller-owned)
 *   X  device fp32 [nb][K], 16-byte aligned;   Y  device fp32 [nb][rows]
 *   nb 1..8;  n_sm: CTAs at most (0: one per SM);  wait_limit_ms: bound of every
 *   wait in the kernel (0: 1000).
 * Asynchronous on `stream`; MK_ERR_UNSUPPORTED for shapes outside the limits,
 * without launching.  mk_matvec_engine_status synchronises `stream` and returns
 * MK_ERR_TIMEOUT if a wait of the last launch ran out. */
mk_status mk_matvec_engine(int32_t engine, const void* W, int32_t rows, int32_t K, const float* X,
                           int32_t nb, float* Y, int32_t n_sm, int32_t wait_limit_ms, void* stream);
mk_status mk_matvec_engine_status(void* stream);

/* Library version string (static storage). */
const char* mk_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MK_H */
