// gdn_internal.h -- host-side launchers of the GDN forward kernels and the
// parameter blocks they take.  Internal to the library (not installed).
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>

namespace gdn {

// Unique id (cuCtxGetId) of the calling thread's current CUDA context; ids are never reused
// within a process, so a context created by a cudaDeviceReset and a later call gets a new one.
// False when no context is current or the driver cannot say.
inline bool current_context_id(unsigned long long *id) {
    typedef CUresult (*GetCurrentFn)(CUcontext *);
    typedef CUresult (*GetIdFn)(CUcontext, unsigned long long *);
    static const auto lookup = [](const char *name) -> void * {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        return p;
    };
    static const GetCurrentFn get_current = reinterpret_cast<GetCurrentFn>(lookup("cuCtxGetCurrent"));
    static const GetIdFn get_id = reinterpret_cast<GetIdFn>(lookup("cuCtxGetId"));
    if (!get_current || !get_id) return false;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}

// Raise a kernel's dynamic shared-memory limit once per CUDA context (the attribute belongs to
// the context's copy of the kernel, so a context re-created by cudaDeviceReset needs it again).
// Safe to call from several host threads (a repeated call only repeats the same attribute set).
constexpr int kMaxDevices = 64;
struct SmemOnce {
    std::atomic<unsigned long long> ctx[kMaxDevices];  // context id it was set in; zero-initialised
};                                                      // (objects of this type are static)
template <typename K>
inline cudaError_t raise_smem_once(SmemOnce &once, K kernel, int bytes) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    unsigned long long id = 0;
    const bool have_id = current_context_id(&id) && id != 0;
    const bool tracked = have_id && dev >= 0 && dev < kMaxDevices;
    if (tracked && once.ctx[dev].load(std::memory_order_acquire) == id) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && tracked) once.ctx[dev].store(id, std::memory_order_release);
    return e;
}

enum class InType { BF16 = 0, F32 = 1, F16 = 2 };

// Kernel launch, optionally with programmatic stream serialization: the kernel
// may then be scheduled while the previous kernel in the stream finishes; it
// must call pdl_wait() before touching that kernel's outputs.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl,
                            const Args &...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Prep: conv4 + SiLU on q, k, v; L2 norm (and the 1/sqrt(d_k) output scale
// folded into q^); log-decay, in-block cumulative log-decay, update gate.
struct PrepParams {
    const void *q, *k, *v;
    long long tok_stride;          // elements between tokens of q, k, v
    const float *g, *b;            // [B][T][H]
    const float *conv_q, *conv_k, *conv_v;  // [H*d][4]
    const float *A_log, *dt_bias;  // [H]
    void *qh, *kh, *vh;            // [B][H][Tp][d]  (fp16 or fp32)
    float *G;                      // [B][H][Tp] in-block (128) inclusive cumsum of log alpha
    float *beta;                   // [B][H][Tp]
    float *log_alpha;              // [B][H][Tp]
    int B, T, H, d, Tp;
    float l2_eps, q_scale;
    int *status;
    unsigned long long wait_limit_ns;
    int rev;                       // reverse scan: internal token t is input token T-1-t
    int debug;                     // GDN_FLAG_DEBUG_CHECKS: index-bounds checks on the stores
};
cudaError_t launch_prep(const PrepParams &p, InType in, bool out_f16, cudaStream_t s);
// Tensor path (16-bit inputs, d = 128): raw tiles staged by TMA through the
// 3-D maps tmq/tmk/tmv over [B][T][H*d] (box {64, 131, 1}).
cudaError_t launch_prep_tma(const PrepParams &p, InType in, const CUtensorMap &tmq, const CUtensorMap &tmk,
                            const CUtensorMap &tmv, cudaStream_t s);

// Intra-block UT transform on tensor cores (d = 128, fp16 operands).  It
// also evaluates the gates of its block from g, b (and writes G, beta, log
// alpha for the scan and the stage tests).
struct ChunkParams {
    const float *g, *bg;            // [B][T][H]
    const float *A_log, *dt_bias;   // [H]
    float *G, *beta, *log_alpha;    // [BH][Tp]
    int T, H;
    __half *W, *U, *Qt, *Kt, *Aqk;  // [BH][Tp][128]
    int BH, Tp, NB;
    int *status;
    unsigned long long wait_limit_ns;
    int rev;                        // reverse scan: block row t holds the gates of input token T-1-t
    int debug;                      // GDN_FLAG_DEBUG_CHECKS: index-bounds checks on the gate accesses
    int save;                       // for the backward: also store T = (I + L)^-1 (through tmT) and
                                    // Aqk's zero upper-right quadrant, so that every Aqk tile is whole
};
cudaError_t launch_chunk(const ChunkParams &p, const CUtensorMap &tmK, const CUtensorMap &tmV,
                         const CUtensorMap &tmQ, const CUtensorMap &tmW, const CUtensorMap &tmU,
                         const CUtensorMap &tmQt, const CUtensorMap &tmAqk, const CUtensorMap &tmAqkH,
                         const CUtensorMap &tmT, cudaStream_t s,
                         bool pdl);  // Kt is written with plain coalesced stores; tmT is read only with save

// Inter-block state scan on tensor cores (d = 128), parallel over segments of
// Ls blocks: pass A (transfer), combine, pass C (outputs + fused output step).
struct ScanParams {
    const float *G;          // [BH][Tp]
    float *Zloc;             // [BH][NS][128][256]: S_loc^T | P^T per segment (pass A)
    float *Sstart;           // [BH][NS][128][128]: S^T at each segment start (combine)
    const void *z;           // [B][T][H][128], token stride tok_stride
    long long tok_stride;
    const float *norm_w;     // [128]
    void *y;                 // [B][T][H][128]
    int out_kind;            // 0 bf16, 1 f32, 2 f16
    float eps;
    int B, T, H, Tp, NB, NS, Ls;
    int *status;
    unsigned long long wait_limit_ns;
    int test_wait_timeout;
    const float *s0;         // [BH][128 (d_v)][128 (d_k)] state before token 0, or null (zero)
    float *s_end;            // [BH][128][128] state after token T-1, or null (not wanted)
    int rev;                 // reverse scan: block row t is z / y token T-1-t
    int debug;               // check that every output value is finite (status word)
    // for the backward (pass C): o itself instead of the normalised, gated output (fp32 into y,
    // out_kind 1), and S^T at the start of every block, fp16 [BH][Tp][128] (block c: rows c*128 ..)
    int raw_o;
    __half *S0b;
    // backward combine: dS^T at every segment end from the backward transfer's local gradients
    const float *Lb;         // [BH][NS][128][128]: local dS^T of each segment (zero at its end)
    float *Sb;               // [BH][NS][128][128]: dS^T at each segment end
};
// pdl: launch with programmatic stream serialization (see launch_k).
cudaError_t launch_transfer(const ScanParams &p, const CUtensorMap &tmW, const CUtensorMap &tmKt,
                            const CUtensorMap &tmU, cudaStream_t s, bool pdl);
cudaError_t launch_combine(const ScanParams &p, cudaStream_t s, bool pdl);
// The combine for the backward: dS^T at each segment end (Sb) from the local gradients (Lb) and the
// forward's transfers (Zloc), last segment first.
cudaError_t launch_combine_bwd(const ScanParams &p, cudaStream_t s, bool pdl);
cudaError_t launch_scan_out(const ScanParams &p, InType zt, const CUtensorMap &tmW, const CUtensorMap &tmQt,
                            const CUtensorMap &tmKt, const CUtensorMap &tmAqk, const CUtensorMap &tmAqkH,
                            const CUtensorMap &tmU, const CUtensorMap &tmZ, cudaStream_t s, bool pdl);

// Fused tensor path (GDN_FLAG_FUSED; 16-bit inputs, d = 128): the transfer and output passes
// over segments of Ls blocks of 64 tokens, each recomputing the preparation and the UT transform
// from the raw inputs, and the combine of the segment states.
struct FusedParams {
    const float *g, *bg;                      // [B][T][H]
    const float *conv_q, *conv_k, *conv_v;    // [H*128][4]
    const float *A_log, *dt_bias, *norm_w;    // [H], [H], [128]
    void *y;                                  // [B][T][H][128], out_kind
    float *SP;                                // [B*H][NS][2][128][128]: S_loc, P of each segment (transfer pass)
    float *SS;                                // [B*H][NS][128][128]: S at each segment start, rows d_v (combine)
    const float *s0;                          // [B*H][128 (d_v)][128 (d_k)] state before token 0, or null (zero)
    float *s_end;                             // [B*H][128][128] state after token T-1, or null
    int B, T, H, NB, NS, Ls;                  // NB = ceil(T / 64) blocks, NS segments of Ls blocks
    float l2_eps, q_scale, eps;
    int rev;                                  // reverse scan: internal token t is input token T-1-t
    int out_kind;                             // y: 0 bf16, 1 f32, 2 f16
    int debug;                                // device-side checks (status word)
    int test_timeout;                         // test hook: one wait that runs out mid-pipeline
    int *status;
    unsigned long long wait_limit_ns;
};
// maps: raw q, k, v [B][T][H*128] boxes {128, 67, 1}; z {128, 64, 1}; y {128, 64, 1} (16-bit
// outputs); y tail {128, T - 64 (NB - 1), 1} (the reverse scan's ragged block).
cudaError_t launch_fused_transfer(const FusedParams &p, InType in, const CUtensorMap *maps, cudaStream_t s, bool pdl);
cudaError_t launch_fused_combine(const FusedParams &p, cudaStream_t s, bool pdl);
cudaError_t launch_fused_output(const FusedParams &p, InType in, const CUtensorMap *maps, cudaStream_t s, bool pdl);

// Sequential fp32 recurrence on CUDA cores (fp32 inputs or d = 64).
struct RecurParams {
    const float *qh, *kh, *vh;  // [B][H][Tp][d]
    const float *log_alpha, *beta;
    float *o;  // [B][T][H][d]
    int B, T, H, d, Tp;
    const float *s0;  // [B*H][d][d] (S[i][j], i over d_v) before token 0, or null (zero)
    float *s_end;     // [B*H][d][d] after token T-1, or null
    int rev;          // reverse scan: internal token t is written to o row T-1-t
};
cudaError_t launch_recurrence(const RecurParams &p, cudaStream_t s);

// y = o / sqrt(mean(o^2) + eps) * w * SiLU(z)
struct OutParams {
    const float *o;  // [B][T][H][dv]
    const void *z;
    long long tok_stride;  // of z
    const float *norm_w;
    void *y;  // [B][T][H][dv]
    int B, T, H, dv;
    float eps;
    int debug;    // check that every output value is finite
    int *status;
};
cudaError_t launch_output(const OutParams &p, InType zt, InType yt, cudaStream_t s);

// Backward (fp32, CUDA cores): the gradient of the forward with respect to
// every input and parameter, for L = sum(y * dy).
struct BwdParams {
    const void *q, *k, *v, *z;      // inputs as in PrepParams / OutParams (token stride tok_stride)
    const void *dy;                 // [B][T][H][d], out dtype, dense
    long long tok_stride;
    const float *g, *bg, *conv_q, *conv_k, *conv_v, *A_log, *dt_bias, *norm_w;
    // the forward, recomputed (prep with fp32 outputs) and kept for the backward
    const float *qh, *kh, *vh, *log_alpha, *beta;  // [BH][Tp][d] / [BH][Tp]
    float *o;                       // [B][T][H][d]
    float *ckpt;                    // [BH][ceil(T/8)][d][d]: the state before every 8th token
    float *dO, *dvh;                // [BH][Tp][d]
    float *dq_part, *dk_part;       // [d/8][BH][Tp][d]: per row-group sums
    float *da_part, *db_part;       // [d/8][BH][Tp]
    float *dnw_part;                // [bwd_out_blocks][d]
    float *dconv_part;              // [B][Tp/64][3][H*d][4]
    float *dA_part, *ddt_part;      // [B][H][Tp/64]
    // results (fp32, dense)
    float *dq, *dk, *dv, *dz;       // [B][T][H][d]
    float *dg, *db;                 // [B][T][H]
    float *dconv_q, *dconv_k, *dconv_v;  // [H*d][4]
    float *dA_log, *ddt_bias;       // [H]
    float *dnorm_w;                 // [d]
    int B, T, H, d, Tp;
    float l2_eps, norm_eps, q_scale;
    // the tensor-core backward: one whole gradient per token in dq_part / dk_part (groups = 1) and
    // d log alpha itself in da_part (tc = 1); dO written as fp16 into dO16 instead of dO
    int groups;
    int tc;
    __half *dO16;
};
int bwd_out_blocks(long long rows);
// The output step backwards (do, dz, norm-weight partials) and the per-token / parameter steps,
// shared by both backward paths.
cudaError_t launch_bwd_out(const BwdParams &p, InType in, InType out, cudaStream_t s);
cudaError_t launch_bwd_tokens(const BwdParams &p, InType in, cudaStream_t s);
cudaError_t launch_bwd_params(const BwdParams &p, cudaStream_t s);

// The backward on tensor cores (16-bit inputs, d = 128), in the block (UT) form, over the forward's
// kept intermediates: a reverse scan of the state gradient dS over segments (transfer pass, combine,
// final pass writing dS^T at every block end), then every block's local gradients.
struct BwdTcParams {
    const float *G, *beta;                 // [BH][Tp]: in-block cumulative log decay, update gate
    const __half *Q, *K, *V;               // q^ (with 1/sqrt(d_k)), k^, v^: [BH][Tp][128]
    const __half *W, *U, *Kt, *Aqk;        // the UT kernel's tiles (Aqk whole)
    const __half *S0b;                     // S^T at every block start (pass C with S0b)
    __half *dSb;                           // dS^T at every block end (the backward's final pass)
    float *dSloc;                          // [BH][NS][128][128]: each segment's dS^T from zero at its end
    const float *dSend;                    // [BH][NS][128][128]: dS^T at each segment end (segments < NS-1)
    float *dqh, *dkh, *dvh;                // [BH][Tp][128]: gradients of Q (q^ with its scale), k^, v^
    float *dla, *dbeta;                    // [BH][Tp]: gradients of log alpha and beta
    int BH, Tp, NB, NS, Ls;
    float q_scale;                         // 1/sqrt(d_k), folded into Q (the per-token step applies it)
    int *status;
    unsigned long long wait_limit_ns;
};
// Reverse pass over the segments (grid: segments x BH).  final = false: segments 1 .. NS-1 from a zero
// gradient at their end, writing dSloc; final = true: every segment from dSend (zero for the last),
// writing dSb.  Tiles: Aqk, dO, Kt, Qt, W ([BH*Tp][128] fp16 maps, {64, 128} boxes, 128-byte swizzle).
cudaError_t launch_bwd_scan(const BwdTcParams &p, bool final_pass, const CUtensorMap &tmAqk,
                            const CUtensorMap &tmDO, const CUtensorMap &tmKt, const CUtensorMap &tmQt,
                            const CUtensorMap &tmW, cudaStream_t s, bool pdl);
// Local gradients of every block (persistent grid); maps as above.
struct BwdTcMaps {
    CUtensorMap S0, W, dO, Aqk, Kt, dS, K, Q, T, U, V;  // V: L2 prefetch only
};
cudaError_t launch_bwd_grad(const BwdTcParams &p, const BwdTcMaps &m, cudaStream_t s, bool pdl);
// Enqueues the five backward kernels after the prep; *launches receives their count.  events
// (optional, 6 cudaEvent_t) are recorded before each launch and after the last.
cudaError_t launch_backward(const BwdParams &p, InType in, InType out, cudaStream_t s, int *launches,
                            void *const *events = nullptr);

}  // namespace gdn

struct gdn_plan_s;
namespace gdn {
// Workspace bytes a plan's forward needs (the value gdn_plan reported).
size_t plan_workspace_bytes(const gdn_plan_s *plan);
}  // namespace gdn

namespace gdn {
// The projections around the core (tcgen05 GEMM, C = A B^T, bf16 operands both K-major, fp32
// accumulation).  mode 0: the input projection x W_in^T, N = 4 H 128 + 2 H columns in the order
// q | k | v | z | g | b, with conv4 + SiLU (+ L2 norm for q, k) in the epilogue; mode 1: the
// output projection y W_out^T.
struct ProjParams {
    int M, N, K;                 // rows (B*T), output columns, reduction (multiple of 64)
    int m_step;                  // rows an M tile advances by (125 in mode 0: 3 history rows)
    int m_tiles, n_tiles;
    int B, T, H, Tp;             // mode 0: batch, tokens, heads, T rounded up to 128
    const float *conv_q, *conv_k, *conv_v;  // [H*128][4], tap 3 on the current token
    __half *qh, *kh, *vh;        // [B][H][Tp][128] fp16 (mode 0)
    __half *z;                   // [B][T][H*128] fp16 (mode 0)
    float *g, *b;                // [B][T][H] fp32 (mode 0)
    float l2_eps, q_scale;
    void *out;                   // [M][N] (mode 1)
    int out_kind;                // 0 bf16, 1 fp32 (mode 1)
    int f16;                     // operands fp16 instead of bf16
    int debug;
    int *status;
    unsigned long long wait_limit_ns;
};
cudaError_t launch_proj(const ProjParams &p, int mode, const CUtensorMap &tmA, const CUtensorMap &tmB,
                        cudaStream_t s, bool pdl);
int proj_m_step(int mode);
// dst[i] = fp16(src[i]) for n bf16 elements (n a multiple of 8; 16-byte aligned pointers).
cudaError_t launch_bf16_to_f16(const void *src, void *dst, size_t n, cudaStream_t s);
int proj_n_tile();

// cuTensorMapEncodeTiled through the runtime's driver entry point (nullptr if unavailable).
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);
EncodeTiledFn encode_fn();

// Layout facts of a tensor-path plan that the block forward needs.
struct PlanLayout {
    int B, T, H, Tp;
    size_t off_status, off_qh, off_kh, off_vh, ws_bytes;
};
bool plan_layout(const gdn_plan_s *plan, PlanLayout *out);

// The tensor path after its prep step: q^, k^, v^ are in the plan's workspace (fp16
// [B][H][Tp][128], zero rows past T); g, b raw gates [B][T][H]; z [B][T][H*128] of type z_type
// with token stride z_stride; y bf16/f16/f32 per the plan.  The status word is not cleared here.
// Returns a gdn_status value.
// events (optional): one cudaEvent_t recorded before each launch, *ev counts them.
// save (optional, for the backward): keep T = (I + L)^-1 and the whole Aqk tiles, write o itself
// (fp32 [B][T][H][128]) instead of y, and S^T at every block start (fp16 [BH][Tp][128]).
struct FwdSave {
    __half *T;
    __half *S0b;
    float *o;
};
int run_tensor_core(const gdn_plan_s *plan, const float *g, const float *b, const float *A_log,
                    const float *dt_bias, const float *norm_w, const void *z, InType z_type,
                    long long z_stride, void *y, void *workspace, cudaStream_t s, bool pdl_first,
                    void *const *events, int *ev, const float *s0, float *s_end,
                    const FwdSave *save = nullptr);
int tensor_core_launches(const gdn_plan_s *plan);
}  // namespace gdn
