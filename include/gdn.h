/*
 * gdn.h -- C ABI of the B200 (sm_100a) Gated DeltaNet forward library.
 *
 * The operation.  The LinMorph project page (Abstract; "Why learn the
 * initialization?") converts softmax self-attention blocks of a video DiT into
 * Gated DeltaNet (GDN) modules built from update gates, decay terms, short
 * convolutions and normalization parameters.  The recurrence is the gated
 * delta rule of "Gated Delta Networks: Improving Mamba2 with Delta Rule"
 * (reference [57] on the VMonarch page, References).  gdn_forward computes,
 * for every batch item b and head h over the frame-major flattened video
 * token sequence t = 0..T-1 (token = f*H_lat*W_lat + y*W_lat + x):
 *
 *   q' = SiLU(conv4(q)), k' = SiLU(conv4(k)), v^ = SiLU(conv4(v))
 *        conv4: causal depthwise kernel-4 convolution over t, tap 3 on the
 *        current token, zero history before t = 0 of each batch item, no bias
 *   q^ = q'/sqrt(|q'|^2 + l2_eps),  k^ = k'/sqrt(|k'|^2 + l2_eps)
 *   alpha_t = exp(-exp(A_log[h]) * softplus(g_t + dt_bias[h])),  beta_t = sigmoid(b_t)
 *   S_t = alpha_t S_{t-1} (I - beta_t k^_t k^_t^T) + beta_t v^_t k^_t^T,  S_{-1} = 0
 *   o_t = S_t q^_t / sqrt(d_k)
 *   y_t = o_t / sqrt(mean(o_t^2) + norm_eps) * norm_w * SiLU(z_t)
 *
 * S is d_v x d_k per (b, h) and is carried in fp32.  The result y is the
 * layer output before the output projection.
 *
 * Precision and range.  With bf16 or f16 inputs and d = 128 the forward runs
 * on the tensor cores: the tensor-core operands (q^, k^, v^, the UT-transform
 * products W, U and the decayed q/k tiles, the fp16 copy of the state and of
 * Delta = U - W S^T) are fp16 with fp32 accumulation; the state itself and
 * every sum stay fp32.  fp16 is chosen over bf16 for its 3 extra mantissa
 * bits; its range ends at 65504.  q^ and k^ are unit vectors and the UT
 * entries are bounded by the gates, so the range that binds is that of
 * v^ = SiLU(conv4(v)), U and the state: inputs whose |conv4(v)| or state
 * entries reach about 6e4 overflow to Inf and give non-finite outputs, which
 * GDN_FLAG_DEBUG_CHECKS reports (activations of 128x unit scale with conv
 * taps of 0.1 are well inside).  For such inputs use the fp32
 * CUDA-core path (GDN_FLAG_FORCE_SIMT).  fp32 inputs, and d = 64, always
 * take that path.
 *
 * Layouts (row-major, element strides):
 *   q, k   [B][T][H][d_k]   token stride tok_stride (elements; 0 = H*d_k)
 *   v, z   [B][T][H][d_v]   token stride tok_stride (0 = H*d_v)
 *   g, b   [B][T][H] fp32
 *   conv_q, conv_k [H*d_k][4] fp32; conv_v [H*d_v][4] fp32 (tap 3 = current token)
 *   A_log, dt_bias [H] fp32;  norm_w [d_v] fp32 (shared by all heads)
 *   y      [B][T][H][d_v], dense, type out_dtype
 * q, k, v, z have type in_dtype.
 *
 * Ownership.  The caller owns every buffer: inputs, output, workspace and
 * staging.  The library allocates no device memory; a plan holds host state
 * only (plus nothing on the device).  All device pointers must be 16-byte
 * aligned and tok_stride * element size must be a multiple of 16 bytes.
 *
 * Errors.  Every call returns a gdn_status; no C++ exception crosses the ABI.
 * gdn_forward validates its arguments on the host and returns
 * GDN_ERR_INVALID_ARG / GDN_ERR_UNSUPPORTED without launching anything.  The
 * launches are asynchronous on the caller's stream: errors the kernels detect
 * on the device (a bounded wait that ran out, a failed debug check) are
 * written to a status word inside the workspace and read back by
 * gdn_get_device_status, which synchronises the stream.
 *
 * Concurrency.  A plan is immutable after gdn_plan and may be shared by
 * threads.  Forwards that may overlap on the GPU need distinct workspaces.
 */
#ifndef GDN_B200_H_
#define GDN_B200_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *gdn_stream_t; /* same type as cudaStream_t; NULL = legacy default stream */

typedef enum {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size or stride, T = 0 with B*H > 0 ... */
    GDN_ERR_UNSUPPORTED = 2,  /* a configuration this build does not implement */
    GDN_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed (launch, copy, tensor map) */
    GDN_ERR_TIMEOUT = 4,      /* a device-side bounded wait ran out (status word) */
    GDN_ERR_DEVICE_CHECK = 5, /* a device-side debug check failed (status word) */
    GDN_ERR_NO_DEVICE = 6     /* no sm_100 device is current */
} gdn_status;

typedef enum {
    GDN_DTYPE_BF16 = 0,
    GDN_DTYPE_F32 = 1,
    GDN_DTYPE_F16 = 2
} gdn_dtype;

/* Plan flags. */
#define GDN_FLAG_DEBUG_CHECKS 0x1u       /* device-side check that every output value of the forward is
                                            finite (a NaN or Inf in the inputs or the arithmetic):
                                            GDN_ERR_DEVICE_CHECK in the status word otherwise */
#define GDN_FLAG_FORCE_SIMT 0x2u         /* use the fp32 CUDA-core path even where the tensor path applies */
#define GDN_FLAG_REVERSE 0x4u            /* reverse (anti-causal) scan: the operation above on the
                                            time-reversed sequence, outputs in the original order.
                                            The state runs from token T-1 down to token 0 (S_{-1} of
                                            gdn_forward_state is the state before token T-1, s_end the
                                            state after token 0), and each conv4 sees the current and
                                            the 3 FOLLOWING tokens, zero past T-1.  The pages leave
                                            the scan direction open (the LinGen page's linear branch
                                            is a bidirectional Mamba2 block); a bidirectional layer is
                                            a forward and a reverse call on the same or separate
                                            parameters, combined by the caller. */
#define GDN_FLAG_FUSED 0x8u              /* tensor path only (ignored elsewhere): the fused forward,
                                            which recomputes the prep and the 64-token UT transform
                                            on chip in two persistent passes (segment transfer,
                                            then scan with the output step) instead of writing the
                                            q^, k^, v^, W, U, Qt, Kt, Aqk intermediates to HBM.
                                            Same results within the tensor path's tolerance; fewer
                                            HBM bytes, but slower on B200 at the documented sizes
                                            (the fused passes are issue-bound), so not the default */
#define GDN_FLAG_TEST_WAIT_TIMEOUT 0x100u /* test hook (tensor path): mid-pipeline, with TMA loads
                                            and tensor-core work in flight, the last kernel waits
                                            on a barrier nothing arrives on, gives up after ~50 ms,
                                            reports GDN_ERR_TIMEOUT in the status word, lets the
                                            work in flight finish and exits; y is then undefined */

typedef struct {
    int B, T, H, d_k, d_v;   /* d_k == d_v, 64 or 128; B, H >= 1; T >= 1 */
    gdn_dtype in_dtype;      /* q, k, v, z */
    gdn_dtype out_dtype;     /* y */
    int conv_size;           /* must be 4 */
    int chunk;               /* UT-transform chunk; must be 64 */
    float l2_eps;            /* inside the sqrt of the q/k L2 norm (1e-6 typical) */
    float norm_eps;          /* inside the sqrt of the output RMSNorm (1e-6 typical) */
    long long tok_stride;    /* elements between consecutive tokens of q,k,v,z; 0 = H*d */
    unsigned flags;          /* GDN_FLAG_* */
} gdn_config;

typedef struct {
    const void *q, *k, *v, *z;                 /* [B][T][H][d] in_dtype, device */
    const float *g, *b;                        /* [B][T][H] fp32, device */
    const float *conv_q, *conv_k, *conv_v;     /* [H*d][4] fp32, device */
    const float *A_log, *dt_bias;              /* [H] fp32, device */
    const float *norm_w;                       /* [d_v] fp32, device */
} gdn_inputs;

typedef struct gdn_plan_s *gdn_plan_t;

/* Validate cfg and build a plan for the current CUDA device.  On success
 * *out receives the plan and *workspace_bytes the size of the device
 * workspace gdn_forward needs (256-byte alignment required).  Host only: no
 * allocation or launch on the device.  Errors: INVALID_ARG (null pointers or
 * invalid sizes), UNSUPPORTED (d not in {64, 128}, d_k != d_v, conv_size != 4,
 * chunk != 64, an output type not in {bf16, f16, f32}), NO_DEVICE. */
gdn_status gdn_plan(const gdn_config *cfg, gdn_plan_t *out, size_t *workspace_bytes);

/* Enqueue the forward on `stream`: y <- GDN(inputs).  Every pointer is a
 * device pointer; workspace has at least *workspace_bytes from gdn_plan.
 * Returns after enqueueing; host-side argument errors return before any
 * launch. */
gdn_status gdn_forward(gdn_plan_t plan, const gdn_inputs *in, void *y, void *workspace,
                       gdn_stream_t stream);

/* gdn_forward with the recurrent state carried in and out, for processing a
 * sequence in pieces (streaming, or a sequence longer than one call).  The
 * recurrence of the gated delta rule (reference [57] on the VMonarch page,
 * References) starts from S_{-1} = s0 instead of zero, and the state after
 * token T-1 is written to s_end:
 *   s0, s_end  [B][H][d_v][d_k] fp32 row-major, S[i][j] with i over d_v and j
 *              over d_k (so that o_t = S_t q^_t); device pointers, 16-byte
 *              aligned, owned by the caller.  s0 = NULL starts from zero (the
 *              result is then bit for bit that of gdn_forward); s_end = NULL
 *              skips the write.  The two must not overlap (ping-pong two
 *              buffers between pieces): INVALID_ARG otherwise.
 * Only the recurrent state is carried.  The short convolutions of each call
 * see zero history before its token 0; a caller that needs the exact
 * continuation of a longer sequence prepends the previous piece's last 3
 * tokens with neutral gates (b = -200, so beta = 0 in fp32 and the state
 * only decays; g = -200 too, so alpha = 1 in fp32 and it does not decay) and
 * drops their 3 outputs.  Same inputs, output, errors and asynchrony as
 * gdn_forward; s_end is complete when the stream reaches the call's end. */
gdn_status gdn_forward_state(gdn_plan_t plan, const gdn_inputs *in, const float *s0, void *y, float *s_end,
                             void *workspace, gdn_stream_t stream);

/* gdn_forward with per-kernel timing: events[i] (a cudaEvent_t the caller
 * created) is recorded on `stream` just before the i-th kernel launch and
 * events[L] after the last one, L = gdn_launches_per_forward(plan);
 * n_events must be L + 1.  Same arguments, errors and result as gdn_forward. */
gdn_status gdn_forward_timed(gdn_plan_t plan, const gdn_inputs *in, void *y, void *workspace,
                             gdn_stream_t stream, void *const *events, int n_events);

/* Bytes of device staging memory gdn_forward_host needs (inputs + output). */
size_t gdn_staging_bytes(gdn_plan_t plan);

/* End-to-end call with HOST buffers: copies every input from host memory
 * (pinned memory recommended) into `staging` (device, gdn_staging_bytes),
 * runs gdn_forward, and copies y back into the host buffer y_host, all
 * enqueued on `stream` (one cudaMemcpyAsync per buffer).  The call returns
 * after enqueueing; synchronise the stream before reading y_host. */
gdn_status gdn_forward_host(gdn_plan_t plan, const gdn_inputs *in_host, void *y_host,
                            void *staging, void *workspace, gdn_stream_t stream);

/* No counterpart in the method's pages: an allocation-free variant of
 * gdn_forward for callers that cannot allocate device memory (code running
 * where cudaMalloc is off limits, or a caller whose device memory is all
 * reserved by a framework and which can hand over only input and output
 * pointers).  The workspace comes from one fixed array of
 * GDN_NOALLOC_SCRATCH_BYTES inside the library's device image, held by every
 * GPU that loads the library until the process exits; no cudaMalloc, cudaFree
 * or allocating library routine is called.  Same inputs, output and result as
 * gdn_forward.  Errors: INVALID_ARG (null plan, inputs or y, or the checks of
 * gdn_forward), UNSUPPORTED when the plan's workspace is larger than
 * GDN_NOALLOC_SCRATCH_BYTES (nothing is enqueued), CUDA if the array's device
 * address cannot be looked up.  The first call in a CUDA context looks that
 * address up (cudaGetSymbolAddress) and caches it with the context's unique
 * id; a call in another context (after cudaDeviceReset, say) looks it up
 * again.  Make the first call on a device, and the first after a reset,
 * before any stream capture.  All calls on a device share the
 * array: calls that may overlap on the GPU (unordered streams, several host
 * threads) race on it; calls on one stream are safe.  The array keeps the last
 * call's contents; the only value that must start at zero, the device status
 * word, is cleared at the start of every call.  Device-side status is not
 * readable through this entry point (it has no workspace pointer to pass to
 * gdn_get_device_status). */
#define GDN_NOALLOC_SCRATCH_BYTES (64ull << 20)
gdn_status gdn_forward_noalloc(gdn_plan_t plan, const gdn_inputs *in, void *y, gdn_stream_t stream);

/* Gradients of L = sum(y * dy) (fp32, dense, device, written not
 * accumulated; caller-owned). */
typedef struct {
    float *dq, *dk, *dv, *dz;            /* [B][T][H][d], 16-byte aligned */
    float *dg, *db;                      /* [B][T][H] */
    float *dconv_q, *dconv_k, *dconv_v;  /* [H*d][4] */
    float *dA_log, *ddt_bias;            /* [H] */
    float *dnorm_w;                      /* [d_v] */
} gdn_grads;

/* Bytes of device workspace gdn_backward needs for this plan (256-byte
 * aligned; a separate size from gdn_forward's).  Tensor-path plans without
 * GDN_FLAG_FUSED: the forward's workspace, then the kept block tiles and
 * states, the state gradients and the per-token gradients
 * (gdn_backward_workspace_offsets).  Other plans: the forward recomputed in
 * fp32, the state every 8 tokens, and per-group partial sums. */
size_t gdn_backward_workspace_bytes(gdn_plan_t plan);

/* Kernel launches one gdn_backward enqueues: 12 (8 with one segment) on the
 * tensor-core backward, 6 otherwise. */
int gdn_backward_launches(gdn_plan_t plan);

/* No counterpart written out in the pages, which train the GDN modules
 * (the LinMorph page: distillation and joint recovery after the weight
 * mapping) without giving the gradient: the gradient of the forward of
 * gdn_forward with respect to every input and parameter, for the loss
 * L = sum(y * dy).  dy is [B][T][H][d_v] of the plan's out_dtype, dense.
 * Plans on the tensor path without GDN_FLAG_FUSED (16-bit inputs, d = 128):
 * on tensor cores, in the block (UT) form of the recurrence.  The forward
 * runs once more keeping its 128-token block tiles (and T = (I + L)^-1, the
 * state at every block start, o); the state gradient dS runs backwards over
 * segments of blocks in parallel (a transfer pass, a combine through the
 * forward's segment transfers, a final pass that writes dS at every block
 * end), then every block's gradients follow from its tiles, S and dS by 16
 * tcgen05 products (fp16 operands, fp32 accumulation), and the per-token
 * steps (L2 norm, SiLU, conv, gates) run in fp32.  Precision: relative L2
 * errors of a few 1e-4 against the exact gradient on N(0,1) inputs (fp16
 * operand rounding, as in the forward); the fp16 range limits of the
 * forward apply to the kept tiles, the states and dL/do.  Other plans (fp32
 * inputs, d = 64, GDN_FLAG_FUSED): fp32 on CUDA cores, the forward
 * recomputed from the inputs, the recurrence's state checkpointed every 8
 * tokens and rebuilt chunk by chunk while its gradient runs backwards.
 * Deterministic on both paths: every sum has a fixed order.
 * Errors: INVALID_ARG (null or misaligned pointers, the workspace checks of
 * gdn_forward), UNSUPPORTED for GDN_FLAG_REVERSE plans; asynchronous on
 * `stream` like gdn_forward. */
gdn_status gdn_backward(gdn_plan_t plan, const gdn_inputs *in, const void *dy, const gdn_grads *grads,
                        void *workspace, gdn_stream_t stream);

/* gdn_backward with per-kernel timing, as gdn_forward_timed: events[i] is
 * recorded before the i-th of the gdn_backward_launches(plan) launches and
 * events[L] after the last; n_events must be L + 1. */
gdn_status gdn_backward_timed(gdn_plan_t plan, const gdn_inputs *in, const void *dy, const gdn_grads *grads,
                              void *workspace, gdn_stream_t stream, void *const *events, int n_events);

/* Synchronise `stream`, then read and clear the device status word in the
 * workspace.  Returns GDN_OK, GDN_ERR_TIMEOUT or GDN_ERR_DEVICE_CHECK (or
 * GDN_ERR_CUDA if the synchronisation itself failed). */
gdn_status gdn_get_device_status(gdn_plan_t plan, void *workspace, gdn_stream_t stream);

/* Number of kernel launches one gdn_forward enqueues for this plan: 3 or 5 on
 * the tensor path (prep, UT transform, [segment transfer, combine,] scan with
 * the output step), 1 or 3 on the fused tensor path ([transfer pass,
 * combine,] output pass), 3 on the CUDA-core path (prep, recurrence,
 * output). */
int gdn_launches_per_forward(gdn_plan_t plan);

/* 1 if the plan runs the tensor-core (tcgen05) path, 0 for the fp32 CUDA-core path. */
int gdn_plan_uses_tensor_path(gdn_plan_t plan);

/* Number of sequence segments the tensor path scans in parallel for each
 * (b, h) (about one scan CTA per SM over all heads); 0 on the CUDA-core path. */
int gdn_plan_segments(gdn_plan_t plan);

/* Introspection for per-stage tests: writes up to n byte offsets, inside the
 * workspace, of the intermediates of the last forward (token rows in scan
 * order: reversed for GDN_FLAG_REVERSE, except o), in this order:
 *   0 status word (int), 1 q^ (scaled by 1/sqrt(d_k)), 2 k^, 3 v^
 *     ([B][H][Tp][d], fp16 on the tensor path, fp32 otherwise; Tp = T rounded
 *     up to 128),
 *   4 G (in-block cumulative log decay), 5 beta, 6 log alpha ([B][H][Tp] fp32),
 *   7 W, 8 U, 9 Qt, 10 Kt, 11 Aqk ([B][H][Tp][128] fp16; tensor path only,
 *     else 0; Aqk is block lower triangular and its upper-right 64x64
 *     quadrant in each 128-row block is never written), 12 o ([B][T][H][d_v] fp32 before the output norm; CUDA-core
 *     path only, else 0), 13 per-segment [S_loc^T | P^T] ([B][H][NS][128][256]
 *     fp32) and 14 segment start states S^T ([B][H][NS][128][128] fp32)
 *     (tensor path without GDN_FLAG_FUSED only, else 0),
 *   15 per-segment [S_loc | P] ([B][H][NS][2][128][128] fp32, S_end =
 *     S_start P + S_loc with the state's d_k index first) and 16 segment
 *     start states ([B][H][NS][128][128] fp32, the same orientation)
 *     (GDN_FLAG_FUSED plans only, else 0; on those plans 1-14 are 0: the
 *     fused forward keeps its other intermediates on chip).
 * Returns the number of offsets written (17 at most). */
int gdn_workspace_offsets(gdn_plan_t plan, size_t *offsets, int n);

/* Byte offsets of the tensor-core backward's own buffers inside the
 * gdn_backward workspace (plans on the tensor path without GDN_FLAG_FUSED;
 * their gdn_backward workspace starts with the forward's layout, at the
 * offsets gdn_workspace_offsets reports), in this order:
 *   0 T = (I + L)^-1 per 128-token block, 1 S^T at every block start
 *     (both [B][H][Tp][128] fp16, block c at rows 128c ..),
 *   2 o before the output norm ([B][T][H][d_v] fp32), 3 dL/do
 *     ([B][H][Tp][128] fp16, zero past T),
 *   4 each segment's local dS^T from zero at its end and 5 dS^T at every
 *     segment end ([B][H][NS][128][128] fp32; 5 unused for the last segment),
 *   6 dS^T at every block end ([B][H][Tp][128] fp16),
 *   7 dL/dQ for Q = q^/sqrt(d_k), 8 dL/dk^, 9 dL/dv^
 *     ([B][H][Tp][128] fp32), 10 dL/d log alpha and 11 dL/d beta
 *     ([B][H][Tp] fp32),
 *   12 norm-weight partial sums, 13 conv-weight partial sums, 14 A_log
 *     partial sums.
 * Returns the number of offsets written (15 at most), 0 for other plans.
 * For tests and profiling: the contents are valid after gdn_backward. */
int gdn_backward_workspace_offsets(gdn_plan_t plan, size_t *offsets, int n);

/* Free a plan (host memory only).  NULL is accepted. */
gdn_status gdn_destroy(gdn_plan_t plan);

/* Static description of a status code. */
const char *gdn_status_string(gdn_status s);

/* ------------------------------------------------------------------------
 * The GDN layer with its projections (gdn_block_*): hidden states in,
 * projected layer output out.  The LinMorph page ("Why learn the
 * initialization?") builds the GDN module's q/k/v/o-side parameters from the
 * attention block's projections; the T3-Video page (Table 1) counts those
 * projections at 7.0T (QKV) and 2.3T (O) MACs for Wan2.1-1.3B at 480x832.
 * For every token row m = b*T + t:
 *   [q | k | v | z | g | b]_m = x_m W_in^T      (W_in: [4*H*d + 2*H][D])
 *   y = the GDN forward above on q, k, v, z, g, b (causal scan)
 *   out_m = y_m W_out^T                          (W_out: [D][H*d])
 * with q, k, v, z [H*d] head-major (head h at columns h*d .. h*d+d-1) and
 * g, b [H].  Operands bf16, fp32 accumulation on the tensor cores.  The
 * input projection runs conv4, SiLU and the q/k L2 norm in its epilogue and
 * hands the prepared operands to the tensor path in fp16 (the projections of
 * q, k, v, z are not rounded to bf16 first); y is stored in bf16 between the
 * scan and the output projection, as the layer's activation type.
 * Requirements: d = 128, H even, D a multiple of 64, B*T < 2^31.
 * Layouts: x [B][T][D] bf16 and out [B][T][D] (bf16 or fp32), dense; the
 * conv, gate and norm parameters as in gdn_inputs.  All pointers device,
 * 16-byte aligned, caller-owned. */
typedef struct {
    int B, T, H, d;          /* d must be 128; H even */
    int D;                   /* model width, a multiple of 64 */
    gdn_dtype out_dtype;     /* out: GDN_DTYPE_BF16 or GDN_DTYPE_F32 */
    float l2_eps, norm_eps;  /* as in gdn_config */
    unsigned flags;          /* GDN_FLAG_DEBUG_CHECKS only */
} gdn_block_config;

typedef struct {
    const void *x;                          /* [B][T][D] bf16 */
    const void *w_in;                       /* [4*H*d + 2*H][D] bf16 (rows: q, k, v, z, g, b) */
    const void *w_out;                      /* [D][H*d] bf16 */
    const float *conv_q, *conv_k, *conv_v;  /* [H*d][4] fp32 */
    const float *A_log, *dt_bias;           /* [H] fp32 */
    const float *norm_w;                    /* [d] fp32 */
} gdn_block_inputs;

typedef struct gdn_block_plan_s *gdn_block_plan_t;

/* Validate cfg and build a block plan for the current device; *workspace_bytes
 * receives the device workspace gdn_block_forward needs (256-byte aligned).
 * Host only.  Errors: INVALID_ARG, UNSUPPORTED (d != 128, odd H, D not a
 * multiple of 64, out_dtype not bf16/f32, flags other than DEBUG_CHECKS),
 * NO_DEVICE. */
gdn_status gdn_block_plan(const gdn_block_config *cfg, gdn_block_plan_t *out, size_t *workspace_bytes);

/* Enqueue the layer on `stream`: out <- (x W_in^T -> GDN -> W_out).  Host
 * argument errors return before any launch; device-side errors go to the
 * status word read by gdn_block_device_status. */
gdn_status gdn_block_forward(gdn_block_plan_t plan, const gdn_block_inputs *in, void *out, void *workspace,
                             gdn_stream_t stream);

/* gdn_block_forward with events[i] recorded before the i-th of its
 * gdn_block_launches(plan) launches and events[L] after the last (n_events
 * must be L + 1); the launches are then not overlapped. */
gdn_status gdn_block_forward_timed(gdn_block_plan_t plan, const gdn_block_inputs *in, void *out, void *workspace,
                                   gdn_stream_t stream, void *const *events, int n_events);

/* Kernel launches of one gdn_block_forward: the input projection, the tensor
 * path's UT transform, [segment transfer, combine,] scan with the output
 * step, and the output projection (4 or 6). */
int gdn_block_launches(gdn_block_plan_t plan);

/* Synchronise `stream`, then read and clear the block workspace's status word
 * (as gdn_get_device_status). */
gdn_status gdn_block_device_status(gdn_block_plan_t plan, void *workspace, gdn_stream_t stream);

/* Free a block plan (host memory only).  NULL is accepted. */
gdn_status gdn_block_destroy(gdn_block_plan_t plan);

#ifdef __cplusplus
}
#endif

#endif /* GDN_B200_H_ */
