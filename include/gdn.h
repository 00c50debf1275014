/*
 * gdn.h — C ABI of libgdn: the Gated DeltaNet (GDN) decode step on NVIDIA B200 (sm_100a).
 *
 * The operation is the single-token (or short multi-token) decode of one GDN
 * linear-attention layer, as dispatched on the page
 * "spark_model/forward/qwen3_5/linear_attention.rs" (Atlas), steps 3 to 8 plus the
 * SiLU(z) gate of the fused steps 9+10+11:
 *
 *   conv   : per channel, a depthwise causal conv of width W over the stored W-1 raw
 *            inputs and the new ones (no bias), SiLU; per-head L2 norm of the Q and K
 *            channels, x / sqrt(sum x^2 + l2_eps); q additionally times q_scale
 *   gate   : g = -exp(A_log) * softplus(a + dt_bias), alpha = exp(g); beta = sigmoid(b)
 *   update : per (sequence, v-head h) with k-head h / (Hv/Hk), FP32 state S[dk][dv]:
 *            S <- alpha S;  S <- S + beta k (v - S^T k)^T;  o = S^T q
 *   norm   : out = o / sqrt(mean_j o_j^2 + rms_eps) * norm_w * silu(z)
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Pointers. Every tensor argument is a DEVICE pointer owned by the caller,
 *   contiguous, row-major in the layout stated, and 16-byte aligned. bf16 values are
 *   passed as their uint16_t bit patterns. The library allocates nothing, keeps no
 *   state between calls and never synchronizes; it only enqueues kernels on `stream`
 *   (a cudaStream_t; NULL means the legacy default stream). Outputs must not alias
 *   inputs or one another.
 * Shapes. Hk = num_k_heads, Hv = num_v_heads (a multiple of Hk, Hv/Hk <= 8),
 *   dk = head_k_dim, dv = head_v_dim (each 16, 32, 64 or 128), W = conv_width (2..8),
 *   C = 2*Hk*dk + Hv*dv qkv channels ordered Q | K | V, head-major inside each block.
 *   B = sequences in this call (B = 0 is a no-op), T = tokens per sequence (1..16),
 *   P = pool_slots.
 * Pools. conv_pool [P][W-1][C] bf16 holds each slot's last W-1 raw (pre-conv) inputs,
 *   row 0 the oldest; state_pool [P][Hv][dk][dv] fp32. Sequence b uses slot slots[b]
 *   of both pools; slots[] (int32, device) must hold distinct values. Pools are
 *   updated in place; slots that no sequence names are never read or written.
 * Multi-token calls (T > 1) are defined as T single-token calls in order.
 * Errors. Every argument check runs on the host before anything is enqueued, so a
 *   call that returns an error has written nothing. Slot VALUES live on the device:
 *   a sequence whose slot is outside [0, P) is skipped entirely (its pools and
 *   outputs untouched) and, when err_flag is non-NULL, the bit
 *   GDN_DEVICE_ERR_SLOT_RANGE is OR-ed into *err_flag (the caller zeroes it; the
 *   library never clears it). Duplicate slots are not detected on the device and
 *   give undefined results; gdn_check_slots_host() checks a host copy. Every wait
 *   inside a kernel is bounded: a CTA whose staged state copy has not landed after
 *   2e9 cycles of its SM's clock (a second at the top clock) gives up, ORs
 *   GDN_DEVICE_ERR_TIMEOUT into *err_flag and writes neither that state tile nor its
 *   outputs (their values are then unspecified).
 *   A failed launch returns GDN_ERR_CUDA.
 */
#ifndef GDN_H_
#define GDN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARGUMENT = 1, /* null pointer, negative size, eps < 0, bad pool size */
    GDN_ERR_UNSUPPORTED = 2,      /* a shape outside the supported set above */
    GDN_ERR_MISALIGNED = 3,       /* a tensor pointer not 16-byte aligned */
    GDN_ERR_SLOT_RANGE = 4,       /* gdn_check_slots_host: slot out of range or repeated */
    GDN_ERR_CUDA = 5              /* the CUDA launch itself failed */
} gdn_status;

/* Bits a kernel ORs into *err_flag. */
#define GDN_DEVICE_ERR_SLOT_RANGE 1 /* a sequence's slot is outside [0, pool_slots) */
#define GDN_DEVICE_ERR_TIMEOUT 2    /* a bounded wait inside the kernel ran out */
#define GDN_DEVICE_ERR_SEQLEN 4     /* a token count (varlen) or accepted count (spec commit) out of range */
#define GDN_DEVICE_ERR_BATCH 8      /* gdn_decode_step_device_batch: *B_dev outside [0, B_max] */

typedef struct {
    int32_t num_k_heads; /* Hk */
    int32_t num_v_heads; /* Hv, a multiple of Hk */
    int32_t head_k_dim;  /* dk */
    int32_t head_v_dim;  /* dv */
    int32_t conv_width;  /* W */
    float l2_eps;        /* q/k L2-norm epsilon (inside the root); the page uses 1e-6 */
    float rms_eps;       /* output RMSNorm epsilon (inside the root) */
    float q_scale;       /* factor on the normalised q; 0 selects 1/sqrt(dk) */
} gdn_config;

/*
 * Stage 1 — step 3 of the page, "fused causal_conv1d_update_l2norm", with the
 * 1/sqrt(d_k) q scale it applies at the kernel output, and the Q|K|V split of step 6.
 *   qkv     [B][T][C] bf16        this call's raw projections
 *   conv_w  [C][W] bf16           tap W-1 multiplies the current token
 *   conv_pool, pool_slots, slots  as above; the slot's history is rolled in place
 *   q_out   [B][T][Hk][dk] fp32   L2-normalised, times q_scale
 *   k_out   [B][T][Hk][dk] fp32   L2-normalised
 *   v_out   [B][T][Hv][dv] fp32   SiLU output, no norm
 *   err_flag nullable device int32
 */
gdn_status gdn_conv_update(const gdn_config* cfg, int32_t B, int32_t T, const uint16_t* qkv,
                           const uint16_t* conv_w, uint16_t* conv_pool, int32_t pool_slots,
                           const int32_t* slots, float* q_out, float* k_out, float* v_out,
                           int32_t* err_flag, void* stream);

/*
 * Stage 2 — steps 4, 5 and 7 of the page: the gate, beta and
 * "gated_delta_rule_decode" on the FP32 state pool, one pass over each state.
 *   q, k    [B][T][Hk][dk] fp32   as produced by gdn_conv_update (q already scaled)
 *   v       [B][T][Hv][dv] fp32
 *   a, b    [B][T][Hv] bf16       raw gate and beta projections
 *   A_log, dt_bias [Hv] fp32
 *   state_pool, pool_slots, slots as above; each named state is read once and
 *                                 written once (after all T tokens)
 *   o       [B][T][Hv][dv] fp32   S^T q with S after the token's update
 */
gdn_status gdn_recurrent_step(const gdn_config* cfg, int32_t B, int32_t T, const float* q,
                              const float* k, const float* v, const uint16_t* a, const uint16_t* b,
                              const float* A_log, const float* dt_bias, float* state_pool,
                              int32_t pool_slots, const int32_t* slots, float* o,
                              int32_t* err_flag, void* stream);

/*
 * Stage 3 — step 8 of the page (per-head RMSNorm over dv with one weight vector
 * shared by all heads) and the SiLU(z) gate of steps 9+10+11.
 *   rows     number of (sequence, token, v-head) rows, i.e. B*T*Hv
 *   o        [rows][dv] fp32
 *   z        [rows][dv] bf16
 *   norm_w   [dv] bf16
 *   out_bf16 [rows][dv] bf16      round-to-nearest-even of the fp32 result
 *   out_f32  [rows][dv] fp32      nullable; the same result before rounding
 */
gdn_status gdn_gated_rmsnorm(const gdn_config* cfg, int32_t rows, const float* o, const uint16_t* z,
                             const uint16_t* norm_w, uint16_t* out_bf16, float* out_f32,
                             void* stream);

/*
 * The fused decode step: the three stages above in ONE kernel launch. Each state
 * tile is streamed from HBM once and written back in place; the conv history of
 * every channel is read and rolled by exactly one CTA; q, k, v, the gates and o
 * never leave the chip.
 *   qkv [B][T][C], a [B][T][Hv], b [B][T][Hv], z [B][T][Hv][dv]   bf16 inputs
 *   conv_w [C][W] bf16, A_log [Hv] fp32, dt_bias [Hv] fp32, norm_w [dv] bf16
 *   conv_pool, state_pool, pool_slots, slots                     as above
 *   out_bf16 [B][T][Hv][dv] bf16
 *   out_f32  [B][T][Hv][dv] fp32, nullable (the unrounded output, for parity checks)
 *   err_flag nullable device int32
 *   workspace nullable device buffer of gdn_decode_workspace_bytes() bytes, zeroed by
 *            the caller once before its first use; every call leaves it zeroed again.
 *            With it, large single-token batches are spread over the SMs dynamically
 *            (faster SMs take more sequences); without it the split is static. The
 *            results are the same bits either way. Calls that may run at the same
 *            time on the GPU need separate workspaces.
 * The first call on a device (per shape) queries the device once and sets a kernel
 * attribute; make it before capturing the call into a CUDA graph.
 * The launch allows programmatic stream serialization: the kernel may begin while the
 * kernel before it in the stream drains, but it reads nothing (inputs, pools, slots,
 * workspace) before that kernel has completed; until then it only issues L2 prefetch
 * hints for the first state tiles it will read.
 */
gdn_status gdn_decode_step(const gdn_config* cfg, int32_t B, int32_t T, const uint16_t* qkv,
                           const uint16_t* a, const uint16_t* b, const uint16_t* z,
                           const uint16_t* conv_w, const float* A_log, const float* dt_bias,
                           const uint16_t* norm_w, uint16_t* conv_pool, float* state_pool,
                           int32_t pool_slots, const int32_t* slots, uint16_t* out_bf16,
                           float* out_f32, int32_t* err_flag, void* workspace, void* stream);

/* Bytes of the optional workspace of gdn_decode_step (a multiple of 16). */
size_t gdn_decode_workspace_bytes(void);

/*
 * gdn_decode_step with the batch count in DEVICE memory, for CUDA-graph replay. The
 * launch is sized for B_max sequences; each kernel reads *B_dev (int32, 4-byte
 * aligned) after the work before it in the stream has completed and processes
 * sequences 0 .. *B_dev - 1 only, exactly as gdn_decode_step with B = *B_dev would
 * (the results may differ from that call in the last bits where B_max selects
 * another kernel than B would). Sequences *B_dev .. B_max - 1: pools and outputs
 * untouched. A captured call therefore serves every batch up to B_max: before each
 * replay write the count to *B_dev and the inputs and slots of that many sequences
 * to the captured buffers (the counterpart of the layer graph hooks on the page
 * "metrale_model_arch/glm5next_dsa/layer.rs", which read the replayed step's
 * positions from device memory). All other arguments are those of gdn_decode_step
 * with B = B_max (tensors sized for B_max). A value of *B_dev outside [0, B_max]
 * runs no sequence and ORs GDN_DEVICE_ERR_BATCH into *err_flag. The host-side
 * kernel choice and device queries happen on the first call per shape: make it
 * before the capture.
 */
gdn_status gdn_decode_step_device_batch(const gdn_config* cfg, const int32_t* B_dev, int32_t B_max, int32_t T,
                                        const uint16_t* qkv, const uint16_t* a, const uint16_t* b, const uint16_t* z,
                                        const uint16_t* conv_w, const float* A_log, const float* dt_bias,
                                        const uint16_t* norm_w, uint16_t* conv_pool, float* state_pool,
                                        int32_t pool_slots, const int32_t* slots, uint16_t* out_bf16, float* out_f32,
                                        int32_t* err_flag, void* workspace, void* stream);

/*
 * The fused decode step for a batch whose sequences bring different numbers of tokens
 * (a chunk of a prompt for some, one token for others) in ONE kernel launch. The
 * pages launch per sequence and have no such layout; each sequence's tokens are
 * processed exactly as gdn_decode_step processes T tokens (steps 3 to 8 and the
 * SiLU(z) gate of steps 9+10+11, the tokens in order, the state on chip in between).
 * The tokens of all sequences are packed row after row:
 *   cu_seqlens [B+1] int32 device, 4-byte aligned: sequence i owns the n_i =
 *            cu_seqlens[i+1] - cu_seqlens[i] rows cu_seqlens[i] .. cu_seqlens[i+1]-1;
 *            cu_seqlens[0] = 0 and cu_seqlens[B] = total_tokens are expected
 *   T_max    the largest n_i, 1..16 (sizes the kernel's on-chip buffers)
 *   total_tokens  rows of the packed tensors (>= 0; only checked on the host)
 *   qkv [total][C], a [total][Hv], b [total][Hv], z [total][Hv][dv]   bf16 inputs
 *   out_bf16 [total][Hv][dv] bf16, out_f32 [total][Hv][dv] fp32 nullable
 *   the weights, pools, slots and err_flag as for gdn_decode_step.
 * A sequence with n_i = 0 is left untouched. A sequence with n_i < 0, n_i > T_max or
 * rows outside [0, total_tokens) is skipped (pools and outputs untouched) and
 * GDN_DEVICE_ERR_SEQLEN is OR-ed into *err_flag; a slot outside [0, pool_slots) is
 * handled as in gdn_decode_step. Rows that no sequence owns are neither read nor
 * written. total_tokens = 0 returns GDN_OK without launching. Launched like
 * gdn_decode_step (programmatic stream serialization, no allocation, no
 * synchronization).
 */
gdn_status gdn_decode_step_varlen(const gdn_config* cfg, int32_t B, const int32_t* cu_seqlens,
                                  int32_t T_max, int32_t total_tokens, const uint16_t* qkv,
                                  const uint16_t* a, const uint16_t* b, const uint16_t* z,
                                  const uint16_t* conv_w, const float* A_log, const float* dt_bias,
                                  const uint16_t* norm_w, uint16_t* conv_pool, float* state_pool,
                                  int32_t pool_slots, const int32_t* slots, uint16_t* out_bf16,
                                  float* out_f32, int32_t* err_flag, void* stream);

/*
 * The projections on either side of the decode step, as GEMMs on the tensor cores
 * (tcgen05, bf16 inputs, fp32 accumulation, bf16 outputs rounded to nearest even).
 * Token rows: rows = B*T <= 256; hidden: the model width, a multiple of 8.
 *
 * gdn_in_proj — step 2 of the page (in_proj_qkv, in_proj_z and the dual-output
 * in_proj_a / in_proj_b, all reading the same normalised input) as ONE GEMM over the
 * four weights stacked row-wise:
 *   x     [rows][hidden] bf16                      the normalised layer input
 *   w_in  [C + Hv*dv + 2*Hv][hidden] bf16          rows: in_proj_qkv (C rows), in_proj_z
 *                                                  (Hv*dv), in_proj_a (Hv), in_proj_b (Hv)
 *   qkv [rows][C], z [rows][Hv*dv], a [rows][Hv], b [rows][Hv] bf16 outputs, laid out as
 *                                                  gdn_decode_step takes them (T = 1 rows,
 *                                                  or [B][T] flattened)
 *   out_f32 [rows][C + Hv*dv + 2*Hv] fp32, nullable: the stacked outputs before rounding
 * gdn_out_proj — the GEMV of the page's fused steps 9+10+11, out = out_proj @ y, on the
 * decode step's output y (already normalised and gated by SiLU(z)):
 *   y     [rows][Hv*dv] bf16, w_out [hidden][Hv*dv] bf16, out [rows][hidden] bf16
 *   out_f32 [rows][hidden] fp32, nullable
 * The first call per shape queries the device (kernel attribute, co-resident clusters,
 * which set how K is split); make it before capturing the call into a CUDA graph.
 * Errors: rows > 256 or hidden not a multiple of 8 give GDN_ERR_UNSUPPORTED; other
 * checks as above, all before anything is enqueued. Every wait inside the kernel is
 * bounded; on expiry GDN_DEVICE_ERR_TIMEOUT is OR-ed into *err_flag (nullable) and
 * the outputs are unspecified. Launched with programmatic stream serialization.
 */
gdn_status gdn_in_proj(const gdn_config* cfg, int32_t hidden, int32_t rows, const uint16_t* x,
                       const uint16_t* w_in, uint16_t* qkv, uint16_t* z, uint16_t* a, uint16_t* b, float* out_f32,
                       int32_t* err_flag, void* stream);
gdn_status gdn_out_proj(const gdn_config* cfg, int32_t hidden, int32_t rows, const uint16_t* y,
                        const uint16_t* w_out, uint16_t* out, float* out_f32, int32_t* err_flag, void* stream);

/*
 * Speculative decoding: verify T drafted tokens, then keep the state after the
 * accepted prefix only. The GDN analogue of the rewind of a rejected speculative
 * draft on the page "metrale_model_arch/glm5next_dsa/layer.rs" (its lockstep check
 * and rewind_to(seq_len) on a rejected draft): a linear-attention state cannot be
 * rewound by truncation, so the verify call leaves both pools as they were and
 * records, per token, the factors of that token's state update; the commit call
 * applies the first n_accept[b] of them.
 *
 * gdn_spec_verify takes the arguments of gdn_decode_step (T = the drafted tokens,
 * 1..16) and writes exactly the outputs a T-token gdn_decode_step would write
 * (steps 3 to 8 and the SiLU(z) gate, the tokens in order), but neither conv_pool nor
 * state_pool is written. Instead, for token t of sequence b:
 *   spec_k     [B][T][Hk][dk] fp32  the normalised key k_t (L2 norm of step 3)
 *   spec_delta [B][T][Hv][dv] fp32  the write delta_t = beta_t (v_t - alpha_t S_{t-1}^T k_t)
 *   spec_alpha [B][T][Hv]     fp32  the decay alpha_t = exp(g_t)
 * so that the state after token t is S_t = alpha_t S_{t-1} + k_t delta_t^T
 * (v-head h uses k-head h / (Hv/Hk)). All three buffers are caller-owned device
 * memory, 16-byte aligned, written in full for every sequence that is not skipped.
 * Skipping (slot out of range) and err_flag are as in gdn_decode_step. Launched
 * like gdn_decode_step (programmatic stream serialization, no allocation).
 */
gdn_status gdn_spec_verify(const gdn_config* cfg, int32_t B, int32_t T, const uint16_t* qkv, const uint16_t* a,
                           const uint16_t* b, const uint16_t* z, const uint16_t* conv_w, const float* A_log,
                           const float* dt_bias, const uint16_t* norm_w, const uint16_t* conv_pool,
                           const float* state_pool, int32_t pool_slots, const int32_t* slots, uint16_t* out_bf16,
                           float* out_f32, float* spec_k, float* spec_delta, float* spec_alpha, int32_t* err_flag,
                           void* stream);

/*
 * Commits the accepted prefix of a gdn_spec_verify call: sequence b keeps its first
 * n = n_accept[b] drafted tokens. Its state becomes S_n (the updates of tokens
 * 0..n-1 applied in order to the state the verify call read) and its conv history
 * becomes the last W-1 raw inputs of [history, qkv tokens 0..n-1], bit for bit. The
 * result equals that of a gdn_decode_step over the first n tokens only.
 *   n_accept   [B] int32 device; 0 leaves the sequence's pools untouched
 *   T          the T of the verify call (the layout of qkv and the spec buffers)
 *   qkv        [B][T][C] bf16, the verify call's input (for the conv history)
 *   spec_k, spec_delta, spec_alpha  as written by the verify call
 *   conv_pool, state_pool, pool_slots, slots  the verify call's pools and slots
 * A sequence whose n_accept is outside [0, T] is skipped and GDN_DEVICE_ERR_SEQLEN
 * is OR-ed into *err_flag; a slot outside [0, pool_slots) is handled as in
 * gdn_decode_step. Each named state is read once and written once (when n > 0).
 */
gdn_status gdn_spec_commit(const gdn_config* cfg, int32_t B, int32_t T, const int32_t* n_accept,
                           const uint16_t* qkv, uint16_t* conv_pool, float* state_pool, int32_t pool_slots,
                           const int32_t* slots, const float* spec_k, const float* spec_delta,
                           const float* spec_alpha, int32_t* err_flag, void* stream);

/*
 * gdn_decode_step for callers that cannot allocate device memory. The pages have
 * no counterpart of this entry point; it exists for the library's users.
 *
 * Some callers cannot provide even the small workspace of gdn_decode_step: code
 * that runs inside a host framework which owns the device allocator, plugins with a
 * fixed memory budget, or latency-critical paths that must not call cudaMalloc
 * (which can synchronize the device). This entry point takes the same arguments as
 * gdn_decode_step without `workspace`, allocates nothing (no cudaMalloc, cudaFree
 * or allocating library call) and uses a fixed scratch array that the library
 * itself places in device memory instead: gdn_decode_static_scratch_bytes() bytes
 * on every GPU that loads the library, held until the process exits.
 *   - The first call on a device looks up that array's device address once (with
 *     the device current); make that first call before any stream capture.
 *   - Each call clears the part of the array it needs with an asynchronous memset
 *     on `stream`, then launches as gdn_decode_step does. The results are the same.
 *   - All calls on a device share the one array, which keeps the last call's
 *     contents: calls that overlap on the GPU (other streams, other threads) race
 *     on it. Serialize them, or use gdn_decode_step with one workspace each.
 *   - If the scratch this build needs exceeds the array, the call returns
 *     GDN_ERR_UNSUPPORTED before doing anything.
 */
gdn_status gdn_decode_step_static_scratch(const gdn_config* cfg, int32_t B, int32_t T,
                                          const uint16_t* qkv, const uint16_t* a,
                                          const uint16_t* b, const uint16_t* z,
                                          const uint16_t* conv_w, const float* A_log,
                                          const float* dt_bias, const uint16_t* norm_w,
                                          uint16_t* conv_pool, float* state_pool,
                                          int32_t pool_slots, const int32_t* slots,
                                          uint16_t* out_bf16, float* out_f32, int32_t* err_flag,
                                          void* stream);

/* Size in bytes of the fixed scratch array of gdn_decode_step_static_scratch. */
size_t gdn_decode_static_scratch_bytes(void);

/*
 * Self-test of the bounded waits inside every kernel of this library (the pages have no
 * counterpart): one GPU thread waits on a barrier phase that nothing completes, gives up
 * after limit_cycles cycles of its SM's clock (1 .. 2^40) and ORs GDN_DEVICE_ERR_TIMEOUT
 * into *err_flag (device int32, required). `cycles` (nullable, device uint64) receives
 * the cycles the wait took. Nothing else is touched; the context stays usable.
 */
gdn_status gdn_selftest_wait_timeout(uint64_t limit_cycles, int32_t* err_flag, uint64_t* cycles, void* stream);

/*
 * Host-side check of a HOST copy of slots[]: GDN_OK when all B values are distinct
 * and in [0, pool_slots), GDN_ERR_SLOT_RANGE otherwise, GDN_ERR_INVALID_ARGUMENT for
 * a null pointer or negative size. Touches no device.
 */
gdn_status gdn_check_slots_host(const int32_t* slots_host, int32_t B, int32_t pool_slots);

/* A static, human-readable name for a status code. */
const char* gdn_status_string(gdn_status status);

/* ABI version of this header: (major << 16) | minor. */
#define GDN_ABI_VERSION ((1 << 16) | 4)
int32_t gdn_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H_ */
