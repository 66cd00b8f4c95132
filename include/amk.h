/*
 * amk.h — C ABI of libamk: batch-1 Llama-family decode as ONE persistent CUDA launch (sm_100a).
 *
 * Source of the operation. "AutoMegaKernel: A Statically-Checked Agent Harness for Self-Retargeting
 * Megakernel Synthesis" (abstract) compiles the whole forward pass of a HuggingFace Llama-family model
 * into a single persistent cooperative kernel for greedy decode, with an int8 weight-only (W8A16)
 * variant; its technical summary ("Problem Statement") fixes the workload as single-stream
 * autoregressive decoding at batch size 1, whose floor is weight bytes / HBM bandwidth, and its
 * "Methodology" (Layer 0) describes one block per SM walking a task order with wait -> dispatch ->
 * signal on monotonic counters. The pages print no API; the calls below are this library's own.
 *
 * Conventions for every call:
 *   - Device pointers are CUDA device addresses on the current device; host pointers are ordinary
 *     host memory. `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *   - The caller owns every buffer it passes (weights, KV cache, logits, token). A handle owns only
 *     what amk_create allocates (task list, counters, scratch, RoPE table, status word) and
 *     amk_destroy frees exactly that.
 *   - Return codes: AMK_OK (0) or a negative AMK_ERR_*. Argument errors are detected on the host
 *     before anything is launched. Launches are asynchronous: a device-side failure (a bounded wait
 *     that ran out) is sticky and is reported by the next amk_decode_step* call and by amk_status.
 *   - Not thread-safe per handle: one handle must not be used from two host threads at once.
 */
#ifndef AMK_H_
#define AMK_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- return codes ---------------------------------------------------------------------------- */
#define AMK_OK                   0
#define AMK_ERR_INVALID_ARG     -1  /* bad pointer, size, alignment, token or position */
#define AMK_ERR_CUDA            -2  /* a CUDA runtime call failed (see amk_last_cuda_error) */
#define AMK_ERR_NOT_RESIDENT    -3  /* the persistent grid cannot be co-resident (1 CTA per SM) */
#define AMK_ERR_DEVICE_TIMEOUT  -4  /* a bounded device wait expired; the handle is unusable */
#define AMK_ERR_UNSUPPORTED     -5  /* dims outside what the kernels support (see amk_create) */
#define AMK_ERR_PLAN            -6  /* the static task-list check rejected the plan */
#define AMK_ERR_NO_MEMORY       -7  /* host or device allocation failed */
#define AMK_ERR_SCRATCH_LIMIT   -8  /* amk_decode_step_noalloc: dims need more than its fixed scratch */

/* ---- enums ----------------------------------------------------------------------------------- */
#define AMK_W_INT8   0   /* int8 weights, one bf16 scale per output row (W8A16) */
#define AMK_W_BF16   1   /* bf16 weights, no scales */
#define AMK_W_INT4   2   /* int4 weights, two per byte, one bf16 scale per output row (W4A16) */

#define AMK_SRC_F32  0   /* packer source element type: fp32 */
#define AMK_SRC_BF16 1   /* packer source element type: bf16 */

/* Weight roles: each selects the packed row order the kernels expect (see amk_pack_weight). */
#define AMK_ROLE_PLAIN    0  /* row-major, rows in source order                                   */
#define AMK_ROLE_QKV      1  /* source = [Wq; Wk; Wv] rows; per head, rows i and i+hd/2 adjacent   */
#define AMK_ROLE_O        2  /* source = Wo [d, Hq*hd], source order                               */
#define AMK_ROLE_GATE_UP  3  /* source = [Wgate; Wup] rows; gate row i and up row i adjacent       */
#define AMK_ROLE_DOWN     4  /* source = Wdown [d, ffn], source order                              */
#define AMK_ROLE_LM_HEAD  5  /* source = lm_head [V, d], source order                              */

/* ---- model description ----------------------------------------------------------------------- */
typedef struct amk_dims {
  int   n_layers;      /* L >= 1                                                              */
  int   d_model;       /* d, a multiple of 64                                                 */
  int   n_q_heads;     /* Hq, a multiple of n_kv_heads                                        */
  int   n_kv_heads;    /* Hkv >= 1; Hq / Hkv in 1..4                                          */
  int   head_dim;      /* hd in {64, 128}                                                     */
  int   ffn;           /* SwiGLU hidden size, a multiple of 64                                */
  int   vocab;         /* V >= 1                                                              */
  int   max_seq;       /* KV cache capacity in positions (>= 1)                               */
  float rope_theta;    /* RoPE base (rotate-half form, no scaling)                            */
  float rms_eps;       /* RMSNorm epsilon                                                     */
  int   weight_dtype;  /* AMK_W_INT8, AMK_W_INT4 or AMK_W_BF16 for every linear weight      */
  int   tied_head;     /* 1: the LM head is the bf16 embedding table; 0: lm_head is given     */
} amk_dims;

/* Device pointers of one model. Per-layer entries are HOST arrays of n_layers DEVICE pointers;
 * amk_create copies the pointer values, so the arrays may be freed after it returns.
 * Packed weights and scales come from amk_pack_weight with the matching role. All device
 * pointers must be 16-byte aligned. */
typedef struct amk_weights {
  const void*        embed;       /* bf16 [V, d]                                            */
  const void* const* attn_norm;   /* [L] bf16 [d]                                           */
  const void* const* ffn_norm;    /* [L] bf16 [d]                                           */
  const void*        final_norm;  /* bf16 [d]                                               */
  const void* const* wqkv;        /* [L] packed AMK_ROLE_QKV,     [(Hq+2Hkv)*hd, d]          */
  const void* const* wo;          /* [L] packed AMK_ROLE_O,       [d, Hq*hd]                 */
  const void* const* wgu;         /* [L] packed AMK_ROLE_GATE_UP, [2*ffn, d]                 */
  const void* const* wdown;       /* [L] packed AMK_ROLE_DOWN,    [d, ffn]                   */
  const void*        lm_head;     /* packed AMK_ROLE_LM_HEAD [V, d]; NULL when tied_head    */
  const void* const* sqkv;        /* [L] bf16 scales in packed row order; NULL for bf16     */
  const void* const* so;
  const void* const* sgu;
  const void* const* sdown;
  const void*        slm;         /* bf16 [V]; NULL when tied_head or bf16                   */
  void*              k_cache;     /* bf16 [L][Hkv][max_seq][hd], read and written            */
  void*              v_cache;     /* bf16 [L][Hkv][max_seq][hd], read and written            */
} amk_weights;

/* Optional tuning and test knobs; pass NULL to amk_create for the defaults (all fields 0). This
 * fourth argument of amk_create is an addition of this library: it carries what the pages' schedule
 * search tunes (skill page, "The ScheduleConfig knobs": tiling.attention.kv_block, SM assignment)
 * plus the wait limit, tracing and one failure-injection hook for tests. */
typedef struct amk_options {
  int grid;              /* persistent CTAs; 0 = one per SM                                    */
  int kv_block;          /* minimum positions per attention chunk; 0 = 64                      */
  int max_kv_chunks;     /* cap on attention chunks per KV head; 0 = min(grid / Hkv, 16) below
                            4096 positions, min(grid / Hkv, 32) from 4096 on                    */
  int timeout_ms;        /* bound on every device wait; 0 = 2000 ms                            */
  int trace;             /* 1: record per-task timestamps (see amk_trace_read)                 */
  int test_drop_signal;  /* TEST ONLY: 1 + index of a counter signal the planner omits, so the
                            waits on it expire with AMK_ERR_DEVICE_TIMEOUT; 0 = off            */
} amk_options;

typedef struct amk_handle amk_handle;

/* ---- packing --------------------------------------------------------------------------------- */

/* Implements the storage of the quantized weight-only variants (technical summary, "Key
 * Contributions", Quantized Megakernels: int8 and int4 weight-only kernels).
 * Bytes of the packed weight buffer for `rows` x `cols` in `dst_dtype` (rows * cols * 1 for int8,
 * * 2 for bf16, / 2 for int4; int4 needs an even `cols`, else 0). */
size_t amk_packed_bytes(int rows, int cols, int dst_dtype);

/* Source row that lands in packed row `packed_row` for `role` (host-only helper, no GPU).
 * Returns -1 on bad arguments. For AMK_ROLE_QKV, within each head of hd rows, packed rows
 * 2i and 2i+1 hold source rows i and i + hd/2; for AMK_ROLE_GATE_UP packed rows 2i and 2i+1
 * hold gate row i (source row i) and up row i (source row ffn + i). */
int amk_packed_row_source(int role, const amk_dims* dims, int rows, int packed_row);

/* Device-side weight packer (W8A16 / W4A16 quantiser, bf16 copier). Implements the int8 (W8A16)
 * and int4 weight-only quantisation the abstract and the technical summary ("Key Contributions",
 * Quantized Megakernels) name; the per-row symmetric scheme is this library's reading of them.
 *   src:        device, [rows, cols] row-major in `src_dtype`; for QKV the rows of Wq, Wk, Wv
 *               stacked, for GATE_UP the rows of Wgate then Wup.
 *   packed_out: device, amk_packed_bytes(rows, cols, dst_dtype) bytes, rows in the role's order.
 *   scales_out: device bf16 [rows] (packed order) for AMK_W_INT8 / AMK_W_INT4; ignored (may be NULL)
 *               for bf16.
 * int8: s = bf16_rne(max|w_row| / 127), q = clamp(rint(w / s), -127, 127); s = 0, q = 0 for a row
 * whose scale rounds to 0. int4: the same with 7 in place of 127; element 2j of a row is the low
 * nibble of byte j and element 2j + 1 the high nibble, each stored as q + 8 (1..15; 8 for q = 0).
 * bf16: round-to-nearest-even of each element.
 * `dims` may be NULL for AMK_ROLE_PLAIN; for other roles rows/cols must match dims.
 * Asynchronous on `stream`. */
int amk_pack_weight(int role, const amk_dims* dims, const void* src, int src_dtype, int rows, int cols,
                    int dst_dtype, void* packed_out, void* scales_out, void* stream);

/* ---- handle lifetime ------------------------------------------------------------------------- */

/* Implements the technical summary's "Methodology", Layer 0 (one persistent block per SM walking a
 * task order with wait -> dispatch -> signal on monotonic counters) and its safety gate (the task
 * list is checked for satisfiable waits, stage order and producer counts before any launch).
 * Validates dims/pointers, builds and statically checks the per-CTA task list, allocates the
 * handle's device state and checks that the persistent grid is co-resident. Synchronous.
 * Supported: head_dim in {64,128}; Hq/Hkv in 1..4; d_model, ffn and Hq*hd multiples of 64 and
 * at most 16384; weight rows of at most 32 KB. On failure *out is NULL. */
int  amk_create(const amk_dims* dims, const amk_weights* weights, const amk_options* options,
                amk_handle** out);

/* Lifetime call of this library (the pages print no API).
 * Frees the handle's own device and host state (never the caller's buffers). Synchronizes the
 * device first. NULL is ignored. */
void amk_destroy(amk_handle* h);

/* ---- the decode step ------------------------------------------------------------------------- */

/* Implements the technical summary's "Problem Statement" (single-stream autoregressive decoding at
 * batch size 1, floor = weight bytes / HBM bandwidth) as the abstract describes it: the whole
 * forward pass of one token in ONE persistent launch, greedy.
 * One greedy decode step in ONE persistent launch on `stream`.
 *   token_id:       token at position `pos`, in [0, V); or -1 to read it from *next_token_out
 *                   (written by the previous step on the same stream: device-side feedback).
 *   pos:            absolute position, 0 <= pos < max_seq. K/V are written at `pos` and attention
 *                   covers positions 0..pos (positions < pos must hold earlier keys/values).
 *   logits_out:     device fp32 [V], or NULL to skip writing logits.
 *   next_token_out: device int32 [1], receives argmax(logits) (lowest index on ties). Required.
 * Returns AMK_ERR_DEVICE_TIMEOUT if an earlier launch of this handle expired a wait. */
int  amk_decode_step(amk_handle* h, int token_id, int pos, float* logits_out, int* next_token_out,
                     void* stream);

/* The conventional execution the technical summary's "Problem Statement" contrasts with (a separate
 * kernel per operator), kept as an ablation.
 * Ablation: the same step with the same device routines, launched one kernel per operation
 * (per layer: QKV, attention partials, attention merge, O, gate/up, down; then LM head and the
 * argmax), so activations cross HBM between kernels and there is no cross-SM counter. */
int  amk_decode_step_unfused(amk_handle* h, int token_id, int pos, float* logits_out,
                             int* next_token_out, void* stream);

/* The pages' rule that an unsafe schedule ends in a clean rejection, never a hung GPU (skill page,
 * "HARD HONESTY RULES"), carried to run time: every device wait is bounded and reports here.
 * Sticky device status without synchronizing: AMK_OK or AMK_ERR_DEVICE_TIMEOUT (a wait expired in
 * an earlier launch). `detail` (may be NULL) receives the raw status word: bits 0..15 the counter
 * or slot index that expired, bits 16..23 the wait kind (1 counter, 2 full slot, 3 empty slot,
 * 4 next-token id out of range at launch, 5 producer waiting for its own copy to land, 6 a tagged
 * input that never became current, 7 shared memory not 1024-byte aligned for the swizzled KV copies). */
int  amk_status(const amk_handle* h, uint32_t* detail);

/* Last CUDA error string seen by this library on this thread ("" if none). */
const char* amk_last_cuda_error(void);

/* ---- decode without device allocation ------------------------------------------------------- */

/* The pages have no counterpart to this call; it is an interface addition of this library.
 * Some callers can't call cudaMalloc: a plugin inside a host framework whose memory pool owns all of
 * the device memory (an outside allocation fails near the pool's limit or is forbidden by policy), or a
 * latency-critical loop where cudaMalloc/cudaFree may synchronize the whole device. amk_create
 * allocates device state, so for them this call does the work of amk_create + amk_decode_step without
 * allocating any device memory: the handle's state (task list, layer pointers, RoPE table, scratch
 * vectors, attention partials, counters) lives in one static device array of 4 MiB inside libamk,
 * resident on every GPU that loads the library until the process exits. It launches the same
 * persistent kernel on the same plan (one CTA per SM, default options) as amk_decode_step.
 *   dims, weights:  as for amk_create (same checks, same ownership: the caller owns every buffer).
 *   token_id, pos, logits_out, next_token_out, stream: as for amk_decode_step.
 * Returns AMK_ERR_SCRATCH_LIMIT, before launching anything, when the dims need more than 4 MiB of state
 * (the task list grows with layers x SMs, the RoPE table with max_seq x head_dim: the 8B-shaped model
 * with 1152 positions needs ~1.8 MiB). The first call on a device (with that device current) looks up
 * the array's device address (cudaGetSymbolAddress) and sets the kernel's attributes; make that first
 * call before any stream capture. Every call shares the array, which keeps the last call's contents:
 * each call zeroes the counters and status words on `stream` and reloads the task list, layer
 * pointers and RoPE table (from pageable host memory) when dims or pointers differ from the previous
 * call on that device; such a reload is refused with AMK_ERR_INVALID_ARG while `stream` is capturing,
 * so every call that changes dims or pointers must also come before any capture. Calls whose
 * launches overlap on the GPU (unordered streams) race on the array and must be serialized by the
 * caller. A wait that expires inside such a launch is not reported, and neither is a next token read
 * back (token_id = -1) that lies outside [0, V): the kernel then decodes token 0 (use
 * amk_decode_step and amk_status for the sticky status). */
int amk_decode_step_noalloc(const amk_dims* dims, const amk_weights* weights, int token_id, int pos,
                            float* logits_out, int* next_token_out, void* stream);

/* ---- plan introspection (host-only) ---------------------------------------------------------- */

typedef struct amk_plan_info {
  int      grid;              /* persistent CTAs                                          */
  int      threads;           /* threads per CTA                                          */
  int      smem_bytes;        /* dynamic shared memory per CTA                            */
  int      n_tasks;           /* tasks over all CTAs                                      */
  int      n_counters;        /* inter-CTA counters                                       */
  int      kv_chunks_max;     /* attention chunks per KV head at most                     */
  uint64_t weight_bytes;      /* weight + scale + embedding-row + gain bytes one step reads */
} amk_plan_info;

int amk_plan_info_get(const amk_handle* h, amk_plan_info* out);

/* The numerator of the technical summary's floor t_min = weight_bytes / HBM_bandwidth ("Problem
 * Statement"), plus the KV bytes a step reads.
 * Bytes one decode step at `pos` must read: weights (+scales), one embedding row, the norm
 * gains and the KV cache over positions 0..pos of every layer. Host-only, no GPU. */
uint64_t amk_step_bytes(const amk_dims* dims, int pos);

/* The safety gate of the technical summary's "Methodology" (deadlock-freedom: satisfiable wait
 * thresholds 1 <= t <= #producers and valid per-SM orders; race-freedom: every producer of a counter
 * in an earlier stage; reachability), run without a GPU.
 * Static task-list check without a GPU: builds the plan for `dims` on `grid` CTAs, optionally
 * plants one defect (mutation 0 = none; 1 drop a signal, 2 raise a wait threshold above its
 * producer count, 3 swap two tasks of one CTA against stage order, 4 make a wait refer to a
 * later stage, 5 drop a stage's producer), runs the checker and writes its verdict to `msg`.
 * Returns AMK_OK when the plan is accepted, AMK_ERR_PLAN when it is rejected. */
int amk_plan_check(const amk_dims* dims, int grid, int mutation, char* msg, int msg_len);

/* ---- tracing --------------------------------------------------------------------------------- */

/* The localisation of the cross-SM synchronisation cost the technical summary's "Experimental
 * Results" (Diagnosis) reports, as per-task timestamps.
 * With options.trace = 1, every CTA records AMK_TRACE_WORDS uint64 per task of the last step:
 *   [0] task word, [1] start, [2] inputs may be read (its counter seen), [3] done, and
 *   %globaltimer stamps (ns) of its phases:
 *   GEMV:      [4] inputs loaded and quantised, [5] first ring slot landed, [6] thread 0's last row
 *              computed, [10] every warp's last row computed, [11] last result block's bulk store
 *              issued, [7] signal issued (after that store completed);
 *   attention: [10] q, k, v staged, [11] first KV slot landed, [4] KV chunk done, [5] partial
 *              issued, [6] ticket taken, [7] head merged and signalled (0 unless this chunk merged
 *              the head; records are not cleared between steps, so compare [7] with [6]);
 *   producer:  [8] the task's first ring item issued, [9] its last item issued;
 *   GEMV inputs: [12] thread 0's input words landed;
 *   every task: [13] and [14] the SM's clock64 at [1] and [3] (so the SM clock during the task).
 * Copies up to `max_records` records into the host buffer `out` (synchronizes the device) and
 * returns how many were written, or a negative code. Record r of CTA b is at index
 * b * (max tasks per CTA) + r; unused records and stamps are zero. The task word holds
 * (op << 32) | (layer << 16) | (index of the task in its CTA's list), op one of: */
#define AMK_TRACE_WORDS 16
#define AMK_OP_QKV  1   /* RMSNorm -> QKV GEMV -> RoPE -> K/V append                         */
#define AMK_OP_ATTN 2   /* attention of one KV head over one KV chunk (+ the head's merge)    */
#define AMK_OP_O    3   /* O GEMV + residual                                                  */
#define AMK_OP_GU   4   /* RMSNorm -> gate/up GEMV -> SwiGLU                                  */
#define AMK_OP_DOWN 5   /* down GEMV + residual                                               */
#define AMK_OP_LM   6   /* final RMSNorm -> LM head -> logits + argmax                        */
int amk_trace_read(amk_handle* h, uint64_t* out, int max_records);

#ifdef __cplusplus
}
#endif
#endif /* AMK_H_ */
