/*
 * gdn.h — C ABI of the B200 (sm_100a) Gated DeltaNet token mixer.
 *
 * The mixer is the linear-attention layer of the Qwen3.8-27B hybrid decoder
 * (Qwen3.8 27B model card, "Gated DeltaNet" bullet): from the projected qkv
 * (10240 channels), z (6144), a and b (48 each) it runs a width-4 depthwise
 * causal conv with silu, L2-normalises q and k, forms the decay
 * g = -exp(A_log) * softplus(a + dt_bias) and the write rate beta = sigmoid(b),
 * runs the gated delta rule on a [128,128] f32 state per value head (16 q/k
 * heads, each read by 3 of the 48 value heads), reads out o = S (q / sqrt(128)),
 * and applies the zero-centred gated RMSNorm o * rsqrt(mean(o^2) + 1e-6) *
 * (1 + w) * silu(z) (same card, "Norms" bullet; Qwen/Qwen3.8-27B architecture
 * page, header table: eps 1e-06).  Each row keeps its conv history and its
 * recurrent state in f32 between calls (same card, cache paragraph).
 *
 * Conventions (readings where the pages are silent):
 *   - qkv channel order [q | k | v], heads contiguous, 128 channels each;
 *   - value head h reads q/k head h / (Vh / Kh);
 *   - conv tap W-1 multiplies the current token, tap 0 the token W-1 back;
 *     no conv bias; missing history is zero;
 *   - state layout [row][value head][v index i][k index j] (row i of S maps
 *     keys to value channel i, so S k is a per-row dot product);
 *   - conv history layout [row][W-1][C], oldest row first, stored as the
 *     exact f32 widening of the bf16 inputs.
 *
 * Memory: every pointer is DEVICE memory owned by the caller, 16-byte
 * aligned, densely packed in the layouts given.  bf16 tensors are passed as
 * uint16_t bit patterns.  The library allocates no device memory and keeps no
 * state between calls other than a per-process cache of driver entry points,
 * two internal streams and a few events per device (created by the first
 * prefill that overlaps its kernels, see gdn_prefill), a device-side error word
 * with the decode kernels' wait bound, and the fixed scratch array of
 * gdn_prefill_noalloc.
 *
 * Streams: `stream` is a cudaStream_t (NULL = the legacy default stream).
 * Every call only enqueues work on it and returns; results are ready when
 * the stream reaches that point.  Calls that share buffers must be ordered
 * by the caller.
 *
 * Errors: functions return GDN_OK (0) or a negative status.  Argument errors
 * are detected on the host before anything is enqueued.  A launch failure
 * returns GDN_ERR_CUDA.  A device-side wait that ran past its limit sets the
 * error word read by gdn_last_device_error(); faults inside a kernel surface
 * as CUDA errors at the caller's next synchronisation.
 */
#ifndef GDN_H_
#define GDN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum gdn_status {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = -1, /* null / misaligned pointer, negative size, bad cu_seqlens */
    GDN_ERR_UNSUPPORTED = -2, /* head_dim != 128, conv_width != 4, Vh % Kh != 0, Vh/Kh > 8, not sm_100 */
    GDN_ERR_CUDA = -3,        /* a CUDA runtime / driver call failed */
    GDN_ERR_WORKSPACE = -4,   /* workspace missing or smaller than the *_workspace_size query */
    GDN_ERR_TIMEOUT = -5      /* a bounded device-side wait expired (see gdn_last_device_error) */
};

typedef struct gdn_dims {
    int32_t num_k_heads; /* Kh: query/key heads (16 in the 27B model) */
    int32_t num_v_heads; /* Vh: value heads (48) */
    int32_t head_dim;    /* D: width of every head (128; the only supported value) */
    int32_t conv_width;  /* W: conv taps (4; the only supported value) */
} gdn_dims;

typedef struct gdn_weights {
    const uint16_t* conv_w; /* bf16 [C][W], C = (2*Kh + Vh) * D, depthwise conv taps */
    const float* A_log;     /* f32 [Vh] */
    const float* dt_bias;   /* f32 [Vh] */
    const float* norm_w;    /* f32 [D], zero-centred: the norm scales by (1 + w) */
} gdn_weights;

/* Bytes of device workspace gdn_prefill needs for B rows of T tokens.
 * Returns 0 for invalid dims. */
size_t gdn_prefill_workspace_size(const gdn_dims* dims, int32_t B, int32_t T);

/*
 * Dense prefill: B rows of T tokens each, all rows at their own state.
 *   qkv  bf16 [B][T][C]         z bf16 [B][T][Vh*D]       a, b bf16 [B][T][Vh]
 *   init_state f32 [B][Vh][D][D] or NULL (zero state)
 *   init_conv  f32 [B][W-1][C]    or NULL (zero history)
 *   out        bf16 [B][T][Vh*D]  gated-norm output, head-major
 *   final_state f32 [B][Vh][D][D] may alias init_state (updated in place)
 *   final_conv  f32 [B][W-1][C]   may alias init_conv
 *   workspace: at least gdn_prefill_workspace_size(dims, B, T) bytes.
 * T = 0 is legal: states and histories are copied through.
 * The prefill computes the recurrence in chunks of 64 tokens (WY form) on
 * tensor cores with f16 operands and f32 accumulation.
 * When the recurrence leaves most SMs idle (few rows of at least 16 chunks;
 * gdn_prefill_schedule reports the plan) the call forks onto internal streams
 * of the device (created on first use) through events recorded on
 * `stream`, and joins back onto `stream` before returning: the work stays
 * ordered on `stream` and can be captured into a CUDA graph.  Concurrent
 * calls from several host threads share those internal streams and run one
 * after the other there.
 */
int gdn_prefill(const gdn_dims* dims, const gdn_weights* w, int32_t B, int32_t T,
                const uint16_t* qkv, const uint16_t* z, const uint16_t* a, const uint16_t* b,
                const float* init_state, const float* init_conv,
                uint16_t* out, float* final_state, float* final_conv,
                void* workspace, size_t workspace_bytes, void* stream);

/*
 * Dense prefill followed by the layer's output projection, in one call: the
 * mixer's gated-norm output y (bf16, kept in the workspace) times out_proj
 * (Qwen/Qwen3.8-27B architecture page, module tree: out_proj 5120x6144):
 *   out[b][t][:] = y[b][t][:] w_out^T      w_out bf16 [hidden][Vh*D], out bf16 [B][T][hidden]
 * Arguments and results otherwise as gdn_prefill (hidden % 8 == 0, else
 * GDN_ERR_UNSUPPORTED).  Workspace: gdn_prefill_out_workspace_size(dims, B, T)
 * bytes (the prefill's workspace plus y).  When the prefill overlaps its
 * kernels (see gdn_prefill_schedule) and its recurrence occupies at most half
 * the SMs, the projection of each recurrence segment's tokens starts on an
 * internal stream of the lowest priority as soon as that segment's outputs are
 * written, while the later segments' recurrence runs; otherwise it runs after
 * the recurrence.  The result is the same, bit for bit, as gdn_prefill followed
 * by gdn_out_proj.
 */
size_t gdn_prefill_out_workspace_size(const gdn_dims* dims, int32_t B, int32_t T);
int gdn_prefill_out(const gdn_dims* dims, const gdn_weights* w, int32_t B, int32_t T, int32_t hidden,
                    const uint16_t* qkv, const uint16_t* z, const uint16_t* a, const uint16_t* b,
                    const float* init_state, const float* init_conv, const uint16_t* w_out, uint16_t* out,
                    float* final_state, float* final_conv, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Schedule of a dense prefill of B rows x T tokens that returns its final
 * state, on the current device: gdn_prefill (from_hidden = 0) or
 * gdn_prefill_hidden (from_hidden = 1).  *segments = S, the number of
 * recurrence segments: S = 1 is the plain schedule on the caller's stream;
 * S > 1 overlaps the WY records of segment s+1 with the recurrence of segment
 * s on internal streams, with segment sizes chosen by a cost model of the
 * kernels.  *launches = the number of kernels one such call launches (2 + 2*S:
 * the load stage or the fused in_proj GEMM, the history writer, S WY and S
 * recurrence launches; one more when gdn_prefill_hidden takes the unfused
 * in_proj).  Both 0 for an empty call.  Returns a
 * status (negative for invalid arguments or an unsupported device).
 * Host-only: enqueues nothing.
 */
int gdn_prefill_schedule(const gdn_dims* dims, int32_t B, int32_t T, int32_t from_hidden, int32_t* segments,
                         int32_t* launches);

/*
 * The same plan for a device with nsm streaming multiprocessors (nsm >= 1,
 * else GDN_ERR_INVALID_ARG), without querying or needing a device: the
 * recurrence runs on CTA pairs when 2 * B * num_v_heads <= nsm, and overlaps
 * only when its CTAs + 32 <= nsm and rows hold at least 16 chunks of 64
 * tokens.  Host-only.
 */
int gdn_prefill_schedule_nsm(const gdn_dims* dims, int32_t B, int32_t T, int32_t from_hidden, int32_t nsm,
                             int32_t* segments, int32_t* launches);

/* Bytes of device workspace gdn_prefill_varlen needs for N rows with
 * total_T tokens in all.  Returns 0 for invalid dims. */
size_t gdn_prefill_varlen_workspace_size(const gdn_dims* dims, int32_t N, int32_t total_T);

/*
 * Packed (variable-length) prefill of N rows ("prefill_slots": a server's
 * rows, each at its own length).  Row n owns tokens [cu[n], cu[n+1]) of the
 * packed tensors.  cu_seqlens_host (host memory) and cu_seqlens_dev (device
 * memory) hold the same N+1 int32 values: cu[0] = 0, non-decreasing,
 * cu[N] = total_T.  The host copy is read during the call for validation and
 * planning; the device copy is read by the kernels.
 *   qkv bf16 [total_T][C], z bf16 [total_T][Vh*D], a, b bf16 [total_T][Vh]
 *   init_state / final_state f32 [N][Vh][D][D], init_conv / final_conv f32
 *   [N][W-1][C], out bf16 [total_T][Vh*D]; aliasing and NULL rules as for
 *   gdn_prefill.  Zero-length rows are legal (state and history copied).
 */
int gdn_prefill_varlen(const gdn_dims* dims, const gdn_weights* w, int32_t N,
                       const int32_t* cu_seqlens_host, const int32_t* cu_seqlens_dev, int32_t total_T,
                       const uint16_t* qkv, const uint16_t* z, const uint16_t* a, const uint16_t* b,
                       const float* init_state, const float* init_conv,
                       uint16_t* out, float* final_state, float* final_conv,
                       void* workspace, size_t workspace_bytes, void* stream);

/*
 * One decode step for `rows` rows ("decode_rows": each row at its own
 * length; GDN has no positional encoding, so a row's position enters only
 * through its state and history).  Every step reads and rewrites each row's
 * f32 state once.
 *   qkv bf16 [rows][C], z bf16 [rows][Vh*D], a, b bf16 [rows][Vh]
 *   state f32 [rows][Vh][D][D]   in/out, updated in place
 *   conv  f32 [rows][W-1][C]     in/out, shifted by one token in place
 *   out   bf16 [rows][Vh*D]
 * rows = 0 is a legal no-op.  No workspace.
 */
int gdn_decode(const gdn_dims* dims, const gdn_weights* w, int32_t rows,
               const uint16_t* qkv, const uint16_t* z, const uint16_t* a, const uint16_t* b,
               float* state, float* conv, uint16_t* out, void* stream);

/*
 * ntok successive decode tokens for each of `rows` rows in one call
 * (verification of speculated tokens, or several new tokens per row): each
 * row's state stays on chip through its ntok sequential updates, so the state
 * is read and written once per call instead of once per token.  Same
 * arithmetic per token as gdn_decode (the same results as ntok calls of it).
 *   qkv bf16 [rows][ntok][C], z bf16 [rows][ntok][Vh*D], a, b bf16 [rows][ntok][Vh]
 *   state f32 [rows][Vh][D][D] and conv f32 [rows][W-1][C] in/out (after the ntok tokens)
 *   out   bf16 [rows][ntok][Vh*D]
 * 1 <= ntok <= 8; GDN_ERR_UNSUPPORTED above 8 or when a q/k head's group of
 * value heads needs more on-chip room for ntok tokens than a block has.
 */
int gdn_decode_multi(const gdn_dims* dims, const gdn_weights* w, int32_t rows, int32_t ntok,
                     const uint16_t* qkv, const uint16_t* z, const uint16_t* a, const uint16_t* b,
                     float* state, float* conv, uint16_t* out, void* stream);

/*
 * Slot-indexed state pool (a server's fixed rows kept in one big buffer).
 * Model card (Qwen3.8 27B, Nestmodels for Linnet), cache paragraph: rows keep
 * their conv history and recurrent state between calls; these two entry
 * points address them through a slot table instead of by batch position.
 *   state_pool f32 [pool_rows][Vh][D][D], conv_pool f32 [pool_rows][W-1][C]
 *   slots_host (host memory) and slots_dev (device memory) hold the same int32
 *   values, one per batch row: batch row r reads and updates pool row
 *   slots[r].  The host copy is checked during the call: every slot in
 *   [0, pool_rows) and no slot twice, else GDN_ERR_INVALID_ARG before anything
 *   is enqueued; the device copy is read by the kernels.  Pool rows that no
 *   slot names are not touched.
 */

/* One decode step of `rows` rows (qkv, z, a, b, out as for gdn_decode),
 * each on pool row slots[r]; the pool rows are updated in place. */
int gdn_decode_slots(const gdn_dims* dims, const gdn_weights* w, int32_t rows,
                     const int32_t* slots_host, const int32_t* slots_dev, int32_t pool_rows,
                     const uint16_t* qkv, const uint16_t* z, const uint16_t* a, const uint16_t* b,
                     float* state_pool, float* conv_pool, uint16_t* out, void* stream);

/* Packed prefill of N rows (cu_seqlens, packed tensors, workspace as for
 * gdn_prefill_varlen with the same workspace size), row n starting from and
 * leaving its state and history in pool row slots[n] (in place).  total_T = 0
 * leaves the pool as it is. */
int gdn_prefill_varlen_slots(const gdn_dims* dims, const gdn_weights* w, int32_t N,
                             const int32_t* cu_seqlens_host, const int32_t* cu_seqlens_dev, int32_t total_T,
                             const int32_t* slots_host, const int32_t* slots_dev, int32_t pool_rows,
                             const uint16_t* qkv, const uint16_t* z, const uint16_t* a, const uint16_t* b,
                             float* state_pool, float* conv_pool, uint16_t* out,
                             void* workspace, size_t workspace_bytes, void* stream);

/*
 * The projections around the mixer as bf16 tensor-core GEMMs with f32
 * accumulation and one rounding to bf16 (Qwen/Qwen3.8-27B architecture page,
 * module tree of `linear_attn`: in_proj_qkv 10240x5120, in_proj_z 6144x5120,
 * in_proj_b and in_proj_a 48x5120, out_proj 5120x6144; row-major weights
 * [out_features][in_features]).
 *   gdn_in_proj:  x bf16 [T][hidden]; w_in bf16 [C + Vh*D + 2*Vh][hidden], the
 *                 rows of in_proj_qkv, in_proj_z, in_proj_b and in_proj_a
 *                 stacked in that order; writes qkv [T][C], z [T][Vh*D],
 *                 b [T][Vh] and a [T][Vh] (the mixer's inputs).
 *   gdn_out_proj: y bf16 [T][Vh*D] (the mixer's output), w_out bf16
 *                 [hidden][Vh*D]; writes out bf16 [T][hidden].
 * The contraction width (hidden, or Vh*D) must be a multiple of 64
 * (GDN_ERR_UNSUPPORTED otherwise); x, y and the weights 16-byte aligned.
 * T = 0 is a legal no-op.  No workspace; asynchronous on `stream`.
 */
int gdn_in_proj(const gdn_dims* dims, int32_t T, int32_t hidden, const uint16_t* x, const uint16_t* w_in,
                uint16_t* qkv, uint16_t* z, uint16_t* b, uint16_t* a, void* stream);
int gdn_out_proj(const gdn_dims* dims, int32_t T, int32_t hidden, const uint16_t* y, const uint16_t* w_out,
                 uint16_t* out, void* stream);

/*
 * Dense prefill from the layer's hidden states: gdn_in_proj and gdn_prefill
 * in one call, with the load stage (conv + silu, q/k L2 norms, gates; model
 * card, "Gated DeltaNet" bullet) computed inside the in_proj GEMM's epilogue,
 * so that qkv, a and b never reach HBM.  Same arithmetic, in the same order,
 * as gdn_in_proj followed by gdn_prefill: the results are bit-identical.
 *   x      bf16 [B*T][hidden] (B rows of T tokens), hidden a multiple of 64
 *   w_in   bf16 [C + Vh*D + 2*Vh][hidden] (as for gdn_in_proj)
 *   init_state, init_conv, out, final_state, final_conv: as for gdn_prefill
 *          (out is the mixer's output, before out_proj; NULL and in-place
 *          rules as there).
 * workspace: gdn_prefill_hidden_workspace_size(dims, B, T) bytes, 16-byte
 * aligned (it also holds z and the rows' staged last tokens).  Head counts
 * whose q/k/v or z widths are not whole 256-column tiles take the unfused pair
 * of launches inside the same call (the workspace size accounts for it).
 * Returns GDN_ERR_UNSUPPORTED for hidden % 64 != 0; otherwise as gdn_prefill.
 */
size_t gdn_prefill_hidden_workspace_size(const gdn_dims* dims, int32_t B, int32_t T);
int gdn_prefill_hidden(const gdn_dims* dims, const gdn_weights* w, int32_t B, int32_t T, int32_t hidden,
                       const uint16_t* x, const uint16_t* w_in, const float* init_state, const float* init_conv,
                       uint16_t* out, float* final_state, float* final_conv, void* workspace,
                       size_t workspace_bytes, void* stream);

/*
 * gdn_prefill_hidden over packed rows (the hidden-state counterpart of
 * gdn_prefill_varlen): x bf16 [total_T][hidden] holds N rows, row n the
 * tokens [cu[n], cu[n+1]); cu_seqlens_host / cu_seqlens_dev, state, history
 * and output layouts, aliasing and NULL rules as for gdn_prefill_varlen
 * (zero-length rows and rows shorter than the conv window are legal).  The
 * same bits as gdn_in_proj followed by gdn_prefill_varlen.  workspace:
 * gdn_prefill_hidden_varlen_workspace_size(dims, N, total_T) bytes.
 */
size_t gdn_prefill_hidden_varlen_workspace_size(const gdn_dims* dims, int32_t N, int32_t total_T);
int gdn_prefill_hidden_varlen(const gdn_dims* dims, const gdn_weights* w, int32_t N,
                              const int32_t* cu_seqlens_host, const int32_t* cu_seqlens_dev, int32_t total_T,
                              int32_t hidden, const uint16_t* x, const uint16_t* w_in, const float* init_state,
                              const float* init_conv, uint16_t* out, float* final_state, float* final_conv,
                              void* workspace, size_t workspace_bytes, void* stream);

/*
 * gdn_prefill without a caller-supplied workspace, for callers that cannot
 * call cudaMalloc: for example a plugin inside an inference engine that owns
 * every device allocation, or a latency-critical path that must not take the
 * implicit device synchronisation of an allocation.  (The pages have no
 * counterpart: this is a deployment convenience of this library.)
 *
 * Same arguments, layouts, aliasing and results as gdn_prefill, minus
 * workspace / workspace_bytes.  The scratch lives in one file-scope device
 * array of GDN_NOALLOC_SCRATCH_BYTES (64 MiB) that every GPU which loads this
 * library holds until the process exits.  A request whose scratch exceeds it
 * (gdn_prefill_workspace_size(dims, B, T) > GDN_NOALLOC_SCRATCH_BYTES) is
 * rejected with GDN_ERR_WORKSPACE before anything is enqueued; for the 27B
 * model's dims (16/48 heads) that is about 1,200 tokens per call (one row of
 * up to 1216 tokens; 29,056 bytes per token plus 1,598,208 bytes per 64-token
 * chunk of a row).  The call itself allocates nothing.
 *
 * The first call on each device resolves the device address of the array
 * (cudaGetSymbolAddress, with that device current); make that first call
 * before any stream capture.  Every call shares the one array and the array
 * keeps the previous call's contents; nothing in it needs to start at zero
 * (every byte is written before it is read within a call).  Calls whose work
 * overlaps on the GPU (different streams, or different host threads without
 * ordering) race on the array: order them on one stream.
 */
#define GDN_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)
int gdn_prefill_noalloc(const gdn_dims* dims, const gdn_weights* w, int32_t B, int32_t T,
                        const uint16_t* qkv, const uint16_t* z, const uint16_t* a, const uint16_t* b,
                        const float* init_state, const float* init_conv,
                        uint16_t* out, float* final_state, float* final_conv, void* stream);

/* Device-side error word of the current device: 0, or the code of the first
 * bounded wait that expired since the last read (GDN_DEVERR_TIMEOUT_COPY: a wait
 * for a bulk copy or for a buffer to be released; GDN_DEVERR_TIMEOUT_MMA: a wait
 * for a tensor-core product).  Cleared by reading.  Synchronises the device. */
#define GDN_DEVERR_TIMEOUT_COPY 1
#define GDN_DEVERR_TIMEOUT_MMA 2
int gdn_last_device_error(void);

/* Bound, in nanoseconds, of every wait inside the decode kernels (gdn_decode,
 * gdn_decode_multi, gdn_decode_slots) on the current device; the default is
 * GDN_DECODE_WAIT_LIMIT_DEFAULT_NS (2 s).  A wait that runs out sets the error
 * word above; the kernel then stops issuing copies, waits (up to 2 s) for the
 * copies it already issued, and returns with its outputs undefined, leaving the
 * context usable.  The kernels that hold tensor memory (prefill, projections)
 * keep a fixed 2 s bound.  Synchronises the device; not for use during stream
 * capture. */
#define GDN_DECODE_WAIT_LIMIT_DEFAULT_NS 2000000000ull
int gdn_set_decode_wait_limit(uint64_t ns);

/* Test hook of the failure path above.  unit >= 0: from then on, in every
 * decode launch on the current device, each CTA's copy producer issues no
 * state copy from the unit-th half-tile of its work onward, so the consumers'
 * wait for that half-tile runs out (after the bound set above) with no copy
 * in flight; -1 (the default) switches it off.  Used with a short bound by the
 * library's tests; never needed otherwise.  Synchronises the device. */
int gdn_test_decode_stop_copies_at(int32_t unit);

/* Human-readable text of a gdn_status value (static storage). */
const char* gdn_status_string(int status);

/* ABI version: major * 10000 + minor * 100 + patch. */
int gdn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H_ */
