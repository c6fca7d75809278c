// gdn_api.cu -- the C ABI declared in include/gdn.h: plan validation and
// workspace layout, tensor-map construction, and the launch sequence of the
// GDN forward.  No device memory is allocated here; every buffer is the
// caller's.
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <new>

#include "gdn.h"
#include "gdn_common.cuh"
#include "gdn_internal.h"

using namespace gdn;

struct gdn_plan_s {
    gdn_config cfg;
    int device;
    bool tensor;
    bool fused;              // GDN_FLAG_FUSED: the two-pass fused forward (64-token blocks)
    int Tp, NB, NS, Ls;      // tensor path: 128-token blocks; fused: 64-token blocks
    long long tok_stride;
    size_t in_esize, out_esize, inter_esize;
    // workspace layout
    size_t off_status, off_qh, off_kh, off_vh, off_G, off_beta, off_la;
    size_t off_W, off_U, off_Qt, off_Kt, off_Aqk, off_Zloc, off_Sstart, off_o, off_SP, off_SS, ws_bytes;
    // backward workspace layout (gdn_backward)
    size_t b_status, b_qh, b_kh, b_vh, b_G, b_beta, b_la, b_o, b_ckpt, b_dO, b_dvh, b_dqp, b_dkp, b_dap, b_dbp,
        b_dnw, b_dconv, b_dA, b_ddt, bws_bytes;
    // the tensor-core backward (tensor plans but fused ones): the forward's layout first, then the
    // kept T and block start states, dO (fp16), the segment-end gradients and dS^T at block ends;
    // b_o, b_dqp / b_dkp / b_dvh (whole dq^ dk^ dv^), b_dap / b_dbp (d log alpha, dbeta) and the
    // partial sums reuse the names above
    bool tc_bwd;
    size_t t_T, t_S0, t_dO16, t_dSloc, t_dSend, t_dSb;
    // staging layout (gdn_forward_host)
    size_t st_q, st_k, st_v, st_z, st_g, st_b, st_cq, st_ck, st_cv, st_A, st_dt, st_nw, st_y, staging_bytes;
};

EncodeTiledFn gdn::encode_fn() {
    // looked up once (function-local statics initialise thread-safely)
    static const EncodeTiledFn fn = []() -> EncodeTiledFn {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<EncodeTiledFn>(ptr);
        cudaGetLastError();
        return nullptr;
    }();
    return fn;
}

namespace {

constexpr unsigned long long kWaitLimitNs = 2000ull * 1000 * 1000;  // 2 s per device-side wait
constexpr int kChunk = 64;  // tokens per block of the fused path

size_t esize(gdn_dtype t) { return t == GDN_DTYPE_F32 ? 4 : 2; }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

InType in_type(gdn_dtype t) {
    return t == GDN_DTYPE_BF16 ? InType::BF16 : (t == GDN_DTYPE_F16 ? InType::F16 : InType::F32);
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// [rows][128] fp16 row-major, loaded as {64, 128} boxes with the 128-byte swizzle.
bool make_tile_map(CUtensorMap *m, void *base, unsigned long long rows, unsigned box_rows = 128) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {128, rows};
    const cuuint64_t strides[1] = {128 * 2};
    const cuuint32_t box[2] = {64, box_rows};
    const cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, base, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Raw activations [B][T][H*d] (token stride tok_stride elements), 16-bit,
// loaded as {box_cols channels, box_rows tokens, 1} boxes without swizzle.
bool make_raw_map(CUtensorMap *m, const void *base, int B, int T, int Hd, long long tok_stride, int box_rows,
                  int box_cols) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(Hd), static_cast<cuuint64_t>(T), static_cast<cuuint64_t>(B)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(tok_stride) * 2,
                                   static_cast<cuuint64_t>(tok_stride) * 2 * static_cast<cuuint64_t>(T)};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows), 1};
    const cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace


size_t gdn::plan_workspace_bytes(const gdn_plan_s *plan) { return plan ? plan->ws_bytes : 0; }

int gdn::run_tensor_core(const gdn_plan_s *plan, const float *g, const float *b, const float *A_log,
                         const float *dt_bias, const float *norm_w, const void *z, InType z_type, long long z_stride,
                         void *y, void *workspace, cudaStream_t s, bool pdl_first, void *const *events, int *ev,
                         const float *s0, float *s_end, const FwdSave *save) {
    const gdn_config &c = plan->cfg;
    const int d = c.d_k;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    int *status = reinterpret_cast<int *>(ws + plan->off_status);
    float *G = reinterpret_cast<float *>(ws + plan->off_G);
    float *beta = reinterpret_cast<float *>(ws + plan->off_beta);
    float *la = reinterpret_cast<float *>(ws + plan->off_la);
    const int rev = (c.flags & GDN_FLAG_REVERSE) ? 1 : 0;
    auto mark = [&]() -> bool {
        if (!events) return true;
        return cudaEventRecord(reinterpret_cast<cudaEvent_t>(events[(*ev)++]), s) == cudaSuccess;
    };
    {
        const unsigned long long rows = static_cast<unsigned long long>(c.B) * c.H * plan->Tp;
        CUtensorMap tmQ, tmK, tmV, tmW, tmU, tmQt, tmKt, tmAqk, tmAqkH;
        if (!make_tile_map(&tmQ, ws + plan->off_qh, rows) || !make_tile_map(&tmK, ws + plan->off_kh, rows) ||
            !make_tile_map(&tmV, ws + plan->off_vh, rows) || !make_tile_map(&tmW, ws + plan->off_W, rows) ||
            !make_tile_map(&tmU, ws + plan->off_U, rows) || !make_tile_map(&tmQt, ws + plan->off_Qt, rows) ||
            !make_tile_map(&tmKt, ws + plan->off_Kt, rows) || !make_tile_map(&tmAqk, ws + plan->off_Aqk, rows) ||
            !make_tile_map(&tmAqkH, ws + plan->off_Aqk, rows, 64))  // Aqk's lower-right quadrant
            return GDN_ERR_CUDA;
        CUtensorMap tmT = tmQt;  // read only when T is kept
        if (save && !make_tile_map(&tmT, save->T, rows)) return GDN_ERR_CUDA;
        ChunkParams cp;
        cp.g = g; cp.bg = b; cp.A_log = A_log; cp.dt_bias = dt_bias;
        cp.G = G; cp.beta = beta; cp.log_alpha = la;
        cp.T = c.T; cp.H = c.H;
        cp.W = reinterpret_cast<__half *>(ws + plan->off_W);
        cp.U = reinterpret_cast<__half *>(ws + plan->off_U);
        cp.Qt = reinterpret_cast<__half *>(ws + plan->off_Qt);
        cp.Kt = reinterpret_cast<__half *>(ws + plan->off_Kt);
        cp.Aqk = reinterpret_cast<__half *>(ws + plan->off_Aqk);
        cp.BH = c.B * c.H; cp.Tp = plan->Tp; cp.NB = plan->NB;
        cp.status = status;
        cp.wait_limit_ns = kWaitLimitNs;
        cp.rev = rev;
        cp.debug = (c.flags & GDN_FLAG_DEBUG_CHECKS) ? 1 : 0;
        cp.save = save ? 1 : 0;
        // The kernels start with programmatic dependent launch (prologue overlapped with the previous
        // kernel's tail), except when per-kernel events are recorded between them.
        const bool pdl = events == nullptr;
        if (!mark() ||
            launch_chunk(cp, tmK, tmV, tmQ, tmW, tmU, tmQt, tmAqk, tmAqkH, tmT, s, pdl && pdl_first) != cudaSuccess)
            return GDN_ERR_CUDA;
        ScanParams sp;
        sp.G = G;
        sp.Zloc = reinterpret_cast<float *>(ws + plan->off_Zloc);
        sp.Sstart = reinterpret_cast<float *>(ws + plan->off_Sstart);
        sp.z = z; sp.tok_stride = z_stride; sp.norm_w = norm_w; sp.y = y;
        sp.out_kind = c.out_dtype == GDN_DTYPE_BF16 ? 0 : (c.out_dtype == GDN_DTYPE_F32 ? 1 : 2);
        sp.eps = c.norm_eps;
        sp.B = c.B; sp.T = c.T; sp.H = c.H; sp.Tp = plan->Tp; sp.NB = plan->NB; sp.NS = plan->NS; sp.Ls = plan->Ls;
        sp.status = status;
        sp.wait_limit_ns = kWaitLimitNs;
        sp.test_wait_timeout = (c.flags & GDN_FLAG_TEST_WAIT_TIMEOUT) ? 1 : 0;
        sp.s0 = s0;
        sp.s_end = s_end;
        sp.rev = rev;
        sp.debug = (c.flags & GDN_FLAG_DEBUG_CHECKS) ? 1 : 0;
        sp.raw_o = 0;
        sp.S0b = nullptr;
        sp.Lb = nullptr;
        sp.Sb = nullptr;
        if (save) {  // o itself (fp32) and the block start states, for the backward
            sp.raw_o = 1;
            sp.y = save->o;
            sp.out_kind = 1;
            sp.S0b = save->S0b;
        }
        if (plan->NS > 1) {
            if (!mark() || launch_transfer(sp, tmW, tmKt, tmU, s, pdl) != cudaSuccess) return GDN_ERR_CUDA;
            if (!mark() || launch_combine(sp, s, pdl) != cudaSuccess) return GDN_ERR_CUDA;
        }
        CUtensorMap tmZ;
        if (!make_raw_map(&tmZ, z, c.B, c.T, c.H * d, z_stride, kBlk, 128)) return GDN_ERR_CUDA;
        if (!mark() || launch_scan_out(sp, z_type, tmW, tmQt, tmKt, tmAqk, tmAqkH, tmU, tmZ, s, pdl) != cudaSuccess)
            return GDN_ERR_CUDA;
        return GDN_OK;
    }
}

int gdn::tensor_core_launches(const gdn_plan_s *plan) { return plan->NS > 1 ? 4 : 2; }

bool gdn::plan_layout(const gdn_plan_s *plan, PlanLayout *out) {
    if (!plan || !out || !plan->tensor || plan->fused) return false;
    out->B = plan->cfg.B; out->T = plan->cfg.T; out->H = plan->cfg.H; out->Tp = plan->Tp;
    out->off_status = plan->off_status; out->off_qh = plan->off_qh; out->off_kh = plan->off_kh;
    out->off_vh = plan->off_vh; out->ws_bytes = plan->ws_bytes;
    return true;
}


extern "C" {

const char *gdn_status_string(gdn_status s) {
    switch (s) {
        case GDN_OK: return "ok";
        case GDN_ERR_INVALID_ARG: return "invalid argument";
        case GDN_ERR_UNSUPPORTED: return "unsupported configuration";
        case GDN_ERR_CUDA: return "CUDA error";
        case GDN_ERR_TIMEOUT: return "device-side wait timed out";
        case GDN_ERR_DEVICE_CHECK: return "device-side check failed";
        case GDN_ERR_NO_DEVICE: return "no sm_100 CUDA device";
    }
    return "unknown status";
}

gdn_status gdn_plan(const gdn_config *cfg, gdn_plan_t *out, size_t *workspace_bytes) {
    if (!cfg || !out || !workspace_bytes) return GDN_ERR_INVALID_ARG;
    *out = nullptr;
    const gdn_config c = *cfg;
    if (c.B < 1 || c.H < 1 || c.T < 1 || c.d_k < 1 || c.d_v < 1) return GDN_ERR_INVALID_ARG;
    if (!(c.l2_eps >= 0.0f) || !(c.norm_eps >= 0.0f) || !isfinite(c.l2_eps) || !isfinite(c.norm_eps))
        return GDN_ERR_INVALID_ARG;
    if (c.in_dtype != GDN_DTYPE_BF16 && c.in_dtype != GDN_DTYPE_F16 && c.in_dtype != GDN_DTYPE_F32)
        return GDN_ERR_UNSUPPORTED;
    if (c.out_dtype != GDN_DTYPE_BF16 && c.out_dtype != GDN_DTYPE_F16 && c.out_dtype != GDN_DTYPE_F32)
        return GDN_ERR_UNSUPPORTED;
    if (c.d_k != c.d_v || (c.d_k != 64 && c.d_k != 128)) return GDN_ERR_UNSUPPORTED;
    if (c.conv_size != 4 || c.chunk != 64) return GDN_ERR_UNSUPPORTED;
    const int d = c.d_k;
    const long long dense = static_cast<long long>(c.H) * d;
    const long long ts = c.tok_stride == 0 ? dense : c.tok_stride;
    if (ts < dense) return GDN_ERR_INVALID_ARG;
    if ((ts * static_cast<long long>(esize(c.in_dtype))) % 16 != 0) return GDN_ERR_INVALID_ARG;
    const long long Tp = (static_cast<long long>(c.T) + kBlk - 1) / kBlk * kBlk;
    const long long BH = static_cast<long long>(c.B) * c.H;
    if (BH * Tp >= (1ll << 31)) return GDN_ERR_UNSUPPORTED;  // TMA row coordinates are int32

    int dev = -1, major = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return GDN_ERR_NO_DEVICE; }
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess || major != 10 ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        return GDN_ERR_NO_DEVICE;
    }

    gdn_plan_s *p = new (std::nothrow) gdn_plan_s;
    if (!p) return GDN_ERR_INVALID_ARG;
    memset(p, 0, sizeof(*p));
    p->cfg = c;
    p->device = dev;
    p->tensor = (c.in_dtype != GDN_DTYPE_F32) && d == 128 && !(c.flags & GDN_FLAG_FORCE_SIMT);
    p->fused = p->tensor && (c.flags & GDN_FLAG_FUSED);
    p->Tp = static_cast<int>(Tp);
    p->NB = static_cast<int>(p->fused ? (static_cast<long long>(c.T) + kChunk - 1) / kChunk : Tp / kBlk);
    // segments: about one scan CTA per SM over all (b, h)
    {
        long long ns = sms / BH;
        if (ns < 1) ns = 1;
        if (ns > p->NB) ns = p->NB;
        p->Ls = static_cast<int>((p->NB + ns - 1) / ns);
        p->NS = (p->NB + p->Ls - 1) / p->Ls;
    }
    p->tok_stride = ts;
    p->in_esize = esize(c.in_dtype);
    p->out_esize = esize(c.out_dtype);
    p->inter_esize = p->tensor ? 2 : 4;

    const size_t A = 1024;
    const size_t nTok = static_cast<size_t>(BH) * Tp;
    const size_t act = nTok * d;
    size_t off = 0;
    p->off_status = off; off = align_up(off + 256, A);
    if (p->fused) {
        const size_t mat = 128 * 128 * 4;
        p->off_SP = off; off = align_up(off + static_cast<size_t>(BH) * p->NS * 2 * mat, A);
        p->off_SS = off; off = align_up(off + static_cast<size_t>(BH) * p->NS * mat, A);
    } else {
        p->off_qh = off; off = align_up(off + act * p->inter_esize, A);
        p->off_kh = off; off = align_up(off + act * p->inter_esize, A);
        p->off_vh = off; off = align_up(off + act * p->inter_esize, A);
        p->off_G = off; off = align_up(off + nTok * 4, A);
        p->off_beta = off; off = align_up(off + nTok * 4, A);
        p->off_la = off; off = align_up(off + nTok * 4, A);
        if (p->tensor) {
            p->off_W = off; off = align_up(off + act * 2, A);
            p->off_U = off; off = align_up(off + act * 2, A);
            p->off_Qt = off; off = align_up(off + act * 2, A);
            p->off_Kt = off; off = align_up(off + act * 2, A);
            p->off_Aqk = off; off = align_up(off + act * 2, A);
            p->off_Zloc = off; off = align_up(off + static_cast<size_t>(BH) * p->NS * 128 * 256 * 4, A);
            p->off_Sstart = off; off = align_up(off + static_cast<size_t>(BH) * p->NS * 128 * 128 * 4, A);
        } else {
            p->off_o = off; off = align_up(off + static_cast<size_t>(c.B) * c.T * c.H * d * 4, A);
        }
    }
    p->ws_bytes = off;

    {  // backward: the forward recomputed in fp32, checkpoints, gradient intermediates and partial sums
        const size_t act4 = nTok * d * 4, tok4 = nTok * 4;
        const size_t G = static_cast<size_t>(d) / 8;
        const size_t NC = (static_cast<size_t>(c.T) + 7) / 8;
        const size_t ntile = static_cast<size_t>(Tp) / 64;
        const size_t nout = static_cast<size_t>(bwd_out_blocks(static_cast<long long>(c.B) * c.T * c.H));
        size_t o2 = 0;
        p->b_status = o2; o2 = align_up(o2 + 256, A);
        p->b_qh = o2; o2 = align_up(o2 + act4, A);
        p->b_kh = o2; o2 = align_up(o2 + act4, A);
        p->b_vh = o2; o2 = align_up(o2 + act4, A);
        p->b_G = o2; o2 = align_up(o2 + tok4, A);
        p->b_beta = o2; o2 = align_up(o2 + tok4, A);
        p->b_la = o2; o2 = align_up(o2 + tok4, A);
        p->b_o = o2; o2 = align_up(o2 + static_cast<size_t>(c.B) * c.T * c.H * d * 4, A);
        p->b_ckpt = o2; o2 = align_up(o2 + static_cast<size_t>(BH) * NC * d * d * 4, A);
        p->b_dO = o2; o2 = align_up(o2 + act4, A);
        p->b_dvh = o2; o2 = align_up(o2 + act4, A);
        p->b_dqp = o2; o2 = align_up(o2 + G * act4, A);
        p->b_dkp = o2; o2 = align_up(o2 + G * act4, A);
        p->b_dap = o2; o2 = align_up(o2 + G * tok4, A);
        p->b_dbp = o2; o2 = align_up(o2 + G * tok4, A);
        p->b_dnw = o2; o2 = align_up(o2 + nout * d * 4, A);
        p->b_dconv = o2; o2 = align_up(o2 + static_cast<size_t>(c.B) * ntile * 3 * c.H * d * 4 * 4, A);
        p->b_dA = o2; o2 = align_up(o2 + static_cast<size_t>(BH) * ntile * 4, A);
        p->b_ddt = o2; o2 = align_up(o2 + static_cast<size_t>(BH) * ntile * 4, A);
        p->bws_bytes = o2;
    }
    p->tc_bwd = p->tensor && !p->fused;
    if (p->tc_bwd) {  // the tensor-core backward's layout (replaces the one above)
        const size_t act2 = nTok * 128 * 2, act4 = nTok * 128 * 4, tok4 = nTok * 4;
        const size_t seg4 = static_cast<size_t>(BH) * p->NS * 128 * 128 * 4;
        const size_t ntile = static_cast<size_t>(Tp) / 64;
        const size_t nout = static_cast<size_t>(bwd_out_blocks(static_cast<long long>(c.B) * c.T * c.H));
        size_t o2 = p->ws_bytes;  // the forward's buffers at their usual offsets (status at 0)
        p->b_status = p->off_status;
        p->t_T = o2; o2 = align_up(o2 + act2, A);
        p->t_S0 = o2; o2 = align_up(o2 + act2, A);
        p->b_o = o2; o2 = align_up(o2 + static_cast<size_t>(c.B) * c.T * c.H * 128 * 4, A);
        p->t_dO16 = o2; o2 = align_up(o2 + act2, A);
        p->t_dSloc = o2; o2 = align_up(o2 + seg4, A);
        p->t_dSend = o2; o2 = align_up(o2 + seg4, A);
        p->t_dSb = o2; o2 = align_up(o2 + act2, A);
        p->b_dqp = o2; o2 = align_up(o2 + act4, A);
        p->b_dkp = o2; o2 = align_up(o2 + act4, A);
        p->b_dvh = o2; o2 = align_up(o2 + act4, A);
        p->b_dap = o2; o2 = align_up(o2 + tok4, A);
        p->b_dbp = o2; o2 = align_up(o2 + tok4, A);
        p->b_dnw = o2; o2 = align_up(o2 + nout * 128 * 4, A);
        p->b_dconv = o2; o2 = align_up(o2 + static_cast<size_t>(c.B) * ntile * 3 * c.H * 128 * 4 * 4, A);
        p->b_dA = o2; o2 = align_up(o2 + static_cast<size_t>(BH) * ntile * 4, A);
        p->b_ddt = o2; o2 = align_up(o2 + static_cast<size_t>(BH) * ntile * 4, A);
        p->bws_bytes = o2;
    }

    const size_t ntok_in = static_cast<size_t>(c.B) * c.T;
    const size_t a_in = ntok_in * c.H * d * p->in_esize;
    off = 0;
    p->st_q = off; off = align_up(off + a_in, 256);
    p->st_k = off; off = align_up(off + a_in, 256);
    p->st_v = off; off = align_up(off + a_in, 256);
    p->st_z = off; off = align_up(off + a_in, 256);
    p->st_g = off; off = align_up(off + ntok_in * c.H * 4, 256);
    p->st_b = off; off = align_up(off + ntok_in * c.H * 4, 256);
    p->st_cq = off; off = align_up(off + static_cast<size_t>(c.H) * d * 16, 256);
    p->st_ck = off; off = align_up(off + static_cast<size_t>(c.H) * d * 16, 256);
    p->st_cv = off; off = align_up(off + static_cast<size_t>(c.H) * d * 16, 256);
    p->st_A = off; off = align_up(off + static_cast<size_t>(c.H) * 4, 256);
    p->st_dt = off; off = align_up(off + static_cast<size_t>(c.H) * 4, 256);
    p->st_nw = off; off = align_up(off + static_cast<size_t>(d) * 4, 256);
    p->st_y = off; off = align_up(off + ntok_in * c.H * d * p->out_esize, 256);
    p->staging_bytes = off;

    *out = p;
    *workspace_bytes = p->ws_bytes;
    return GDN_OK;
}

gdn_status gdn_destroy(gdn_plan_t plan) {
    delete plan;
    return GDN_OK;
}

int gdn_launches_per_forward(gdn_plan_t plan) {
    if (!plan) return 0;
    if (!plan->tensor) return 3;          // prep, recurrence, output
    if (plan->fused) return plan->NS > 1 ? 3 : 1;  // [transfer pass, combine,] output pass
    return plan->NS > 1 ? 5 : 3;          // prep, chunk, [transfer, combine,] scan+output
}

int gdn_plan_uses_tensor_path(gdn_plan_t plan) { return plan && plan->tensor ? 1 : 0; }

int gdn_plan_segments(gdn_plan_t plan) { return plan && plan->tensor ? plan->NS : 0; }

size_t gdn_staging_bytes(gdn_plan_t plan) { return plan ? plan->staging_bytes : 0; }

int gdn_workspace_offsets(gdn_plan_t plan, size_t *offsets, int n) {
    if (!plan || !offsets || n <= 0) return 0;
    const size_t all[17] = {plan->off_status, plan->off_qh, plan->off_kh, plan->off_vh, plan->off_G,
                            plan->off_beta, plan->off_la, plan->off_W, plan->off_U, plan->off_Qt,
                            plan->off_Kt, plan->off_Aqk, plan->off_o, plan->off_Zloc, plan->off_Sstart,
                            plan->off_SP, plan->off_SS};
    const int m = n < 17 ? n : 17;
    for (int i = 0; i < m; ++i) offsets[i] = all[i];
    return m;
}

int gdn_backward_workspace_offsets(gdn_plan_t plan, size_t *offsets, int n) {
    if (!plan || !offsets || n <= 0 || !plan->tc_bwd) return 0;
    const size_t all[15] = {plan->t_T,    plan->t_S0,   plan->b_o,   plan->t_dO16, plan->t_dSloc,
                            plan->t_dSend, plan->t_dSb, plan->b_dqp, plan->b_dkp,  plan->b_dvh,
                            plan->b_dap,  plan->b_dbp,  plan->b_dnw, plan->b_dconv, plan->b_dA};
    const int m = n < 15 ? n : 15;
    for (int i = 0; i < m; ++i) offsets[i] = all[i];
    return m;
}

static gdn_status forward_impl(gdn_plan_t plan, const gdn_inputs *in, void *y, void *workspace,
                               gdn_stream_t stream, void *const *events, const float *s0 = nullptr,
                               float *s_end = nullptr) {
    if (!plan || !in || !y || !workspace) return GDN_ERR_INVALID_ARG;
    const gdn_config &c = plan->cfg;
    if ((s0 && !aligned16(s0)) || (s_end && !aligned16(s_end))) return GDN_ERR_INVALID_ARG;
    if (s0 && s_end) {  // the end state is written while other CTAs may still read the initial one
        const size_t bytes = static_cast<size_t>(c.B) * c.H * c.d_v * c.d_k * sizeof(float);
        const uintptr_t a = reinterpret_cast<uintptr_t>(s0), e = reinterpret_cast<uintptr_t>(s_end);
        if (a < e + bytes && e < a + bytes) return GDN_ERR_INVALID_ARG;
    }
    const void *ptrs16[] = {in->q, in->k, in->v, in->z, y};
    for (const void *q : ptrs16)
        if (!q || !aligned16(q)) return GDN_ERR_INVALID_ARG;
    const void *ptrs4[] = {in->g, in->b, in->conv_q, in->conv_k, in->conv_v, in->A_log, in->dt_bias, in->norm_w};
    for (const void *q : ptrs4)
        if (!q || (reinterpret_cast<uintptr_t>(q) & 3u)) return GDN_ERR_INVALID_ARG;
    const void *ptrsw[] = {in->conv_q, in->conv_k, in->conv_v};
    for (const void *q : ptrsw)
        if (!aligned16(q)) return GDN_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return GDN_ERR_INVALID_ARG;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != plan->device) return GDN_ERR_INVALID_ARG;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    int *status = reinterpret_cast<int *>(ws + plan->off_status);
    float *G = reinterpret_cast<float *>(ws + plan->off_G);
    float *beta = reinterpret_cast<float *>(ws + plan->off_beta);
    float *la = reinterpret_cast<float *>(ws + plan->off_la);
    float *o = reinterpret_cast<float *>(ws + plan->off_o);
    const int d = c.d_k;

    if (cudaMemsetAsync(status, 0, sizeof(int), s) != cudaSuccess) return GDN_ERR_CUDA;
    int ev = 0;
    auto mark = [&]() -> bool {
        if (!events) return true;
        return cudaEventRecord(reinterpret_cast<cudaEvent_t>(events[ev++]), s) == cudaSuccess;
    };

    const int rev = (c.flags & GDN_FLAG_REVERSE) ? 1 : 0;
    if (plan->fused) {
        // raw q, k, v boxes of 64 tokens + 3 of conv history; z and y boxes of 64 tokens; the
        // reverse scan's ragged last block stores only its T - 64 (NB - 1) live rows
        CUtensorMap maps[6];
        const int Hd = c.H * d;
        const int tail = c.T - kChunk * (plan->NB - 1);
        if (!make_raw_map(&maps[0], in->q, c.B, c.T, Hd, plan->tok_stride, kChunk + 3, 128) ||
            !make_raw_map(&maps[1], in->k, c.B, c.T, Hd, plan->tok_stride, kChunk + 3, 128) ||
            !make_raw_map(&maps[2], in->v, c.B, c.T, Hd, plan->tok_stride, kChunk + 3, 128) ||
            !make_raw_map(&maps[3], in->z, c.B, c.T, Hd, plan->tok_stride, kChunk, 128))
            return GDN_ERR_CUDA;
        if (c.out_dtype != GDN_DTYPE_F32) {
            if (!make_raw_map(&maps[4], y, c.B, c.T, Hd, Hd, kChunk, 128) ||
                !make_raw_map(&maps[5], y, c.B, c.T, Hd, Hd, tail, 128))
                return GDN_ERR_CUDA;
        } else {
            maps[4] = maps[3];  // not used: fp32 outputs are stored directly
            maps[5] = maps[3];
        }
        FusedParams fp;
        fp.g = in->g; fp.bg = in->b;
        fp.conv_q = in->conv_q; fp.conv_k = in->conv_k; fp.conv_v = in->conv_v;
        fp.A_log = in->A_log; fp.dt_bias = in->dt_bias; fp.norm_w = in->norm_w;
        fp.y = y;
        fp.SP = reinterpret_cast<float *>(ws + plan->off_SP);
        fp.SS = reinterpret_cast<float *>(ws + plan->off_SS);
        fp.s0 = s0;
        fp.s_end = s_end;
        fp.B = c.B; fp.T = c.T; fp.H = c.H; fp.NB = plan->NB; fp.NS = plan->NS; fp.Ls = plan->Ls;
        fp.l2_eps = c.l2_eps;
        fp.q_scale = 1.0f / sqrtf(static_cast<float>(d));
        fp.eps = c.norm_eps;
        fp.rev = rev;
        fp.out_kind = c.out_dtype == GDN_DTYPE_BF16 ? 0 : (c.out_dtype == GDN_DTYPE_F32 ? 1 : 2);
        fp.debug = (c.flags & GDN_FLAG_DEBUG_CHECKS) ? 1 : 0;
        fp.test_timeout = (c.flags & GDN_FLAG_TEST_WAIT_TIMEOUT) ? 1 : 0;
        fp.status = status;
        fp.wait_limit_ns = kWaitLimitNs;
        // The kernels after the first start with programmatic dependent launch (prologue overlapped
        // with the previous kernel), except when per-kernel events are recorded between them.
        const bool pdl = events == nullptr;
        const InType it = in_type(c.in_dtype);
        if (plan->NS > 1) {
            if (!mark() || launch_fused_transfer(fp, it, maps, s, false) != cudaSuccess) return GDN_ERR_CUDA;
            if (!mark() || launch_fused_combine(fp, s, pdl) != cudaSuccess) return GDN_ERR_CUDA;
        }
        if (!mark() || launch_fused_output(fp, it, maps, s, plan->NS > 1 && pdl) != cudaSuccess) return GDN_ERR_CUDA;
        if (!mark()) return GDN_ERR_CUDA;
        return GDN_OK;
    }

    PrepParams pp;
    pp.q = in->q; pp.k = in->k; pp.v = in->v;
    pp.tok_stride = plan->tok_stride;
    pp.g = in->g; pp.b = in->b;
    pp.conv_q = in->conv_q; pp.conv_k = in->conv_k; pp.conv_v = in->conv_v;
    pp.A_log = in->A_log; pp.dt_bias = in->dt_bias;
    pp.qh = ws + plan->off_qh; pp.kh = ws + plan->off_kh; pp.vh = ws + plan->off_vh;
    pp.G = G; pp.beta = beta; pp.log_alpha = la;
    pp.B = c.B; pp.T = c.T; pp.H = c.H; pp.d = d; pp.Tp = plan->Tp;
    pp.l2_eps = c.l2_eps;
    pp.q_scale = 1.0f / sqrtf(static_cast<float>(d));
    pp.status = status;
    pp.wait_limit_ns = kWaitLimitNs;
    pp.rev = rev;
    pp.debug = (c.flags & GDN_FLAG_DEBUG_CHECKS) ? 1 : 0;
    if (plan->tensor) {
        CUtensorMap rq, rk, rv;
        if (!make_raw_map(&rq, in->q, c.B, c.T, c.H * d, plan->tok_stride, 64 + 3, 128) ||
            !make_raw_map(&rk, in->k, c.B, c.T, c.H * d, plan->tok_stride, 64 + 3, 128) ||
            !make_raw_map(&rv, in->v, c.B, c.T, c.H * d, plan->tok_stride, 64 + 3, 128))
            return GDN_ERR_CUDA;
        if (!mark() || launch_prep_tma(pp, in_type(c.in_dtype), rq, rk, rv, s) != cudaSuccess) return GDN_ERR_CUDA;
    } else if (!mark() || launch_prep(pp, in_type(c.in_dtype), false, s) != cudaSuccess) {
        return GDN_ERR_CUDA;
    }

    if (plan->tensor) {
        const int st = run_tensor_core(plan, in->g, in->b, in->A_log, in->dt_bias, in->norm_w, in->z,
                                       in_type(c.in_dtype), plan->tok_stride, y, workspace, s, events == nullptr,
                                       events, &ev, s0, s_end);
        if (st != GDN_OK) return static_cast<gdn_status>(st);
        if (!mark()) return GDN_ERR_CUDA;
        return GDN_OK;
    } else {
        RecurParams rp;
        rp.qh = reinterpret_cast<const float *>(ws + plan->off_qh);
        rp.kh = reinterpret_cast<const float *>(ws + plan->off_kh);
        rp.vh = reinterpret_cast<const float *>(ws + plan->off_vh);
        rp.log_alpha = la; rp.beta = beta; rp.o = o;
        rp.B = c.B; rp.T = c.T; rp.H = c.H; rp.d = d; rp.Tp = plan->Tp;
        rp.s0 = s0; rp.s_end = s_end; rp.rev = rev;
        if (!mark() || launch_recurrence(rp, s) != cudaSuccess) return GDN_ERR_CUDA;
    }

    OutParams op;
    op.o = o; op.z = in->z; op.tok_stride = plan->tok_stride; op.norm_w = in->norm_w; op.y = y;
    op.B = c.B; op.T = c.T; op.H = c.H; op.dv = c.d_v; op.eps = c.norm_eps;
    op.debug = (c.flags & GDN_FLAG_DEBUG_CHECKS) ? 1 : 0;
    op.status = status;
    if (!mark() || launch_output(op, in_type(c.in_dtype), in_type(c.out_dtype), s) != cudaSuccess)
        return GDN_ERR_CUDA;
    if (!mark()) return GDN_ERR_CUDA;
    return GDN_OK;
}

gdn_status gdn_forward(gdn_plan_t plan, const gdn_inputs *in, void *y, void *workspace, gdn_stream_t stream) {
    return forward_impl(plan, in, y, workspace, stream, nullptr);
}

gdn_status gdn_forward_state(gdn_plan_t plan, const gdn_inputs *in, const float *s0, void *y, float *s_end,
                             void *workspace, gdn_stream_t stream) {
    return forward_impl(plan, in, y, workspace, stream, nullptr, s0, s_end);
}

gdn_status gdn_forward_timed(gdn_plan_t plan, const gdn_inputs *in, void *y, void *workspace,
                             gdn_stream_t stream, void *const *events, int n_events) {
    if (!plan || !events || n_events != gdn_launches_per_forward(plan) + 1) return GDN_ERR_INVALID_ARG;
    for (int i = 0; i < n_events; ++i)
        if (!events[i]) return GDN_ERR_INVALID_ARG;
    return forward_impl(plan, in, y, workspace, stream, events);
}

gdn_status gdn_forward_host(gdn_plan_t plan, const gdn_inputs *in_host, void *y_host, void *staging,
                            void *workspace, gdn_stream_t stream) {
    if (!plan || !in_host || !y_host || !staging || !workspace) return GDN_ERR_INVALID_ARG;
    const gdn_config &c = plan->cfg;
    const int d = c.d_k;
    if (plan->tok_stride != static_cast<long long>(c.H) * d) return GDN_ERR_UNSUPPORTED;  // host buffers are dense
    if (reinterpret_cast<uintptr_t>(staging) & 255u) return GDN_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *st = static_cast<uint8_t *>(staging);
    const size_t ntok = static_cast<size_t>(c.B) * c.T;
    const size_t a_in = ntok * c.H * d * plan->in_esize;
    const size_t gb = ntok * c.H * 4;
    const size_t cw = static_cast<size_t>(c.H) * d * 16;
    struct Copy { size_t off; const void *src; size_t bytes; } copies[] = {
        {plan->st_q, in_host->q, a_in}, {plan->st_k, in_host->k, a_in}, {plan->st_v, in_host->v, a_in},
        {plan->st_z, in_host->z, a_in}, {plan->st_g, in_host->g, gb}, {plan->st_b, in_host->b, gb},
        {plan->st_cq, in_host->conv_q, cw}, {plan->st_ck, in_host->conv_k, cw}, {plan->st_cv, in_host->conv_v, cw},
        {plan->st_A, in_host->A_log, static_cast<size_t>(c.H) * 4},
        {plan->st_dt, in_host->dt_bias, static_cast<size_t>(c.H) * 4},
        {plan->st_nw, in_host->norm_w, static_cast<size_t>(d) * 4}};
    for (const Copy &cp : copies) {
        if (!cp.src) return GDN_ERR_INVALID_ARG;
        if (cudaMemcpyAsync(st + cp.off, cp.src, cp.bytes, cudaMemcpyHostToDevice, s) != cudaSuccess)
            return GDN_ERR_CUDA;
    }
    gdn_inputs dev;
    dev.q = st + plan->st_q; dev.k = st + plan->st_k; dev.v = st + plan->st_v; dev.z = st + plan->st_z;
    dev.g = reinterpret_cast<const float *>(st + plan->st_g);
    dev.b = reinterpret_cast<const float *>(st + plan->st_b);
    dev.conv_q = reinterpret_cast<const float *>(st + plan->st_cq);
    dev.conv_k = reinterpret_cast<const float *>(st + plan->st_ck);
    dev.conv_v = reinterpret_cast<const float *>(st + plan->st_cv);
    dev.A_log = reinterpret_cast<const float *>(st + plan->st_A);
    dev.dt_bias = reinterpret_cast<const float *>(st + plan->st_dt);
    dev.norm_w = reinterpret_cast<const float *>(st + plan->st_nw);
    const gdn_status rc = gdn_forward(plan, &dev, st + plan->st_y, workspace, stream);
    if (rc != GDN_OK) return rc;
    if (cudaMemcpyAsync(y_host, st + plan->st_y, ntok * c.H * d * plan->out_esize, cudaMemcpyDeviceToHost, s) !=
        cudaSuccess)
        return GDN_ERR_CUDA;
    return GDN_OK;
}

size_t gdn_backward_workspace_bytes(gdn_plan_t plan) { return plan ? plan->bws_bytes : 0; }

int gdn_backward_launches(gdn_plan_t plan) {
    if (!plan) return 0;
    // tensor-core backward: prep, the forward with its intermediates kept (UT, [transfer, combine,]
    // output pass), the output step backwards, [the backward transfer and combine,] the final
    // backward pass, the block gradients, the per-token and parameter steps
    if (plan->tc_bwd) return plan->NS > 1 ? 12 : 8;
    return 6;  // prep + the five fp32 backward kernels
}

// The tensor-core backward: the forward with its intermediates kept, the output step backwards,
// the reverse scan of the state gradient over segments, every block's local gradients, then the
// per-token (L2 norm, SiLU, conv, gates) and parameter steps.
static gdn_status backward_tc(gdn_plan_t plan, const gdn_inputs *in, const void *dy, const gdn_grads *gr, uint8_t *ws,
                              cudaStream_t s, void *const *events) {
    const gdn_config &c = plan->cfg;
    const int d = c.d_k;
    int *status = reinterpret_cast<int *>(ws + plan->off_status);
    auto F = [&](size_t off) { return reinterpret_cast<float *>(ws + off); };
    auto H16 = [&](size_t off) { return reinterpret_cast<__half *>(ws + off); };
    int ev = 0;
    auto mark = [&]() -> bool {
        if (!events) return true;
        return cudaEventRecord(reinterpret_cast<cudaEvent_t>(events[ev++]), s) == cudaSuccess;
    };
    const float q_scale = 1.0f / sqrtf(static_cast<float>(d));
    const unsigned long long rows = static_cast<unsigned long long>(c.B) * c.H * plan->Tp;
    const int BH = c.B * c.H;

    // ---- forward (prep, UT transform, segment scan), keeping T, the block start states and o
    PrepParams pp;
    memset(&pp, 0, sizeof(pp));
    pp.q = in->q; pp.k = in->k; pp.v = in->v;
    pp.tok_stride = plan->tok_stride;
    pp.g = in->g; pp.b = in->b;
    pp.conv_q = in->conv_q; pp.conv_k = in->conv_k; pp.conv_v = in->conv_v;
    pp.A_log = in->A_log; pp.dt_bias = in->dt_bias;
    pp.qh = ws + plan->off_qh; pp.kh = ws + plan->off_kh; pp.vh = ws + plan->off_vh;
    pp.G = F(plan->off_G); pp.beta = F(plan->off_beta); pp.log_alpha = F(plan->off_la);
    pp.B = c.B; pp.T = c.T; pp.H = c.H; pp.d = d; pp.Tp = plan->Tp;
    pp.l2_eps = c.l2_eps;
    pp.q_scale = q_scale;
    pp.status = status;
    pp.wait_limit_ns = kWaitLimitNs;
    {
        CUtensorMap rq, rk, rv;
        if (!make_raw_map(&rq, in->q, c.B, c.T, c.H * d, plan->tok_stride, 64 + 3, 128) ||
            !make_raw_map(&rk, in->k, c.B, c.T, c.H * d, plan->tok_stride, 64 + 3, 128) ||
            !make_raw_map(&rv, in->v, c.B, c.T, c.H * d, plan->tok_stride, 64 + 3, 128))
            return GDN_ERR_CUDA;
        if (!mark() || launch_prep_tma(pp, in_type(c.in_dtype), rq, rk, rv, s) != cudaSuccess) return GDN_ERR_CUDA;
    }
    FwdSave save;
    save.T = H16(plan->t_T);
    save.S0b = H16(plan->t_S0);
    save.o = F(plan->b_o);
    const int st = run_tensor_core(plan, in->g, in->b, in->A_log, in->dt_bias, in->norm_w, in->z, in_type(c.in_dtype),
                                   plan->tok_stride, nullptr, ws, s, true, events, &ev, nullptr, nullptr, &save);
    if (st != GDN_OK) return static_cast<gdn_status>(st);

    // ---- the output step backwards: dO (fp16, zero on padding rows), dz, norm-weight partials
    BwdParams bp;
    memset(&bp, 0, sizeof(bp));
    bp.q = in->q; bp.k = in->k; bp.v = in->v; bp.z = in->z; bp.dy = dy;
    bp.tok_stride = plan->tok_stride;
    bp.g = in->g; bp.bg = in->b; bp.conv_q = in->conv_q; bp.conv_k = in->conv_k; bp.conv_v = in->conv_v;
    bp.A_log = in->A_log; bp.dt_bias = in->dt_bias; bp.norm_w = in->norm_w;
    bp.log_alpha = F(plan->off_la);
    bp.o = F(plan->b_o);
    bp.dO16 = H16(plan->t_dO16);
    bp.dvh = F(plan->b_dvh);
    bp.dq_part = F(plan->b_dqp); bp.dk_part = F(plan->b_dkp); bp.da_part = F(plan->b_dap); bp.db_part = F(plan->b_dbp);
    bp.dnw_part = F(plan->b_dnw); bp.dconv_part = F(plan->b_dconv); bp.dA_part = F(plan->b_dA);
    bp.ddt_part = F(plan->b_ddt);
    bp.dq = gr->dq; bp.dk = gr->dk; bp.dv = gr->dv; bp.dz = gr->dz; bp.dg = gr->dg; bp.db = gr->db;
    bp.dconv_q = gr->dconv_q; bp.dconv_k = gr->dconv_k; bp.dconv_v = gr->dconv_v;
    bp.dA_log = gr->dA_log; bp.ddt_bias = gr->ddt_bias; bp.dnorm_w = gr->dnorm_w;
    bp.B = c.B; bp.T = c.T; bp.H = c.H; bp.d = d; bp.Tp = plan->Tp;
    bp.l2_eps = c.l2_eps; bp.norm_eps = c.norm_eps; bp.q_scale = q_scale;
    bp.groups = 1;
    bp.tc = 1;
    if (plan->Tp > c.T &&
        cudaMemset2DAsync(bp.dO16 + static_cast<size_t>(c.T) * 128, static_cast<size_t>(plan->Tp) * 256, 0,
                          static_cast<size_t>(plan->Tp - c.T) * 256, BH, s) != cudaSuccess)
        return GDN_ERR_CUDA;
    if (!mark() || launch_bwd_out(bp, in_type(c.in_dtype), in_type(c.out_dtype), s) != cudaSuccess) return GDN_ERR_CUDA;

    // ---- reverse scan of dS: transfer pass, combine, final pass (dS^T at every block end)
    CUtensorMap tmAqk, tmDO, tmKt, tmQt, tmW;
    if (!make_tile_map(&tmAqk, ws + plan->off_Aqk, rows) || !make_tile_map(&tmDO, bp.dO16, rows) ||
        !make_tile_map(&tmKt, ws + plan->off_Kt, rows) || !make_tile_map(&tmQt, ws + plan->off_Qt, rows) ||
        !make_tile_map(&tmW, ws + plan->off_W, rows))
        return GDN_ERR_CUDA;
    BwdTcParams tp;
    memset(&tp, 0, sizeof(tp));
    tp.G = F(plan->off_G); tp.beta = F(plan->off_beta);
    tp.Q = H16(plan->off_qh); tp.K = H16(plan->off_kh); tp.V = H16(plan->off_vh);
    tp.W = H16(plan->off_W); tp.U = H16(plan->off_U); tp.Kt = H16(plan->off_Kt); tp.Aqk = H16(plan->off_Aqk);
    tp.S0b = save.S0b;
    tp.dSb = H16(plan->t_dSb);
    tp.dSloc = F(plan->t_dSloc);
    tp.dSend = F(plan->t_dSend);
    tp.dqh = bp.dq_part; tp.dkh = bp.dk_part; tp.dvh = bp.dvh;
    tp.dla = bp.da_part; tp.dbeta = bp.db_part;
    tp.BH = BH; tp.Tp = plan->Tp; tp.NB = plan->NB; tp.NS = plan->NS; tp.Ls = plan->Ls;
    tp.q_scale = q_scale;
    tp.status = status;
    tp.wait_limit_ns = kWaitLimitNs;
    const bool pdl = events == nullptr;
    if (plan->NS > 1) {
        if (!mark() || launch_bwd_scan(tp, false, tmAqk, tmDO, tmKt, tmQt, tmW, s, pdl) != cudaSuccess)
            return GDN_ERR_CUDA;
        ScanParams sp;
        memset(&sp, 0, sizeof(sp));
        sp.Zloc = F(plan->off_Zloc);
        sp.Lb = tp.dSloc;
        sp.Sb = F(plan->t_dSend);
        sp.B = c.B; sp.T = c.T; sp.H = c.H; sp.Tp = plan->Tp; sp.NB = plan->NB; sp.NS = plan->NS; sp.Ls = plan->Ls;
        sp.status = status;
        sp.wait_limit_ns = kWaitLimitNs;
        if (!mark() || launch_combine_bwd(sp, s, pdl) != cudaSuccess) return GDN_ERR_CUDA;
    }
    if (!mark() || launch_bwd_scan(tp, true, tmAqk, tmDO, tmKt, tmQt, tmW, s, pdl && plan->NS > 1) != cudaSuccess)
        return GDN_ERR_CUDA;

    // ---- every block's local gradients
    BwdTcMaps mp;
    if (!make_tile_map(&mp.S0, save.S0b, rows) || !make_tile_map(&mp.W, ws + plan->off_W, rows) ||
        !make_tile_map(&mp.dO, bp.dO16, rows) || !make_tile_map(&mp.Aqk, ws + plan->off_Aqk, rows) ||
        !make_tile_map(&mp.Kt, ws + plan->off_Kt, rows) || !make_tile_map(&mp.dS, tp.dSb, rows) ||
        !make_tile_map(&mp.K, ws + plan->off_kh, rows) || !make_tile_map(&mp.Q, ws + plan->off_qh, rows) ||
        !make_tile_map(&mp.T, save.T, rows) || !make_tile_map(&mp.U, ws + plan->off_U, rows) ||
        !make_tile_map(&mp.V, ws + plan->off_vh, rows))
        return GDN_ERR_CUDA;
    if (!mark() || launch_bwd_grad(tp, mp, s, pdl) != cudaSuccess) return GDN_ERR_CUDA;

    // ---- per token (L2 norm, SiLU and conv backwards, gates) and the parameter sums
    if (!mark() || launch_bwd_tokens(bp, in_type(c.in_dtype), s) != cudaSuccess) return GDN_ERR_CUDA;
    if (!mark() || launch_bwd_params(bp, s) != cudaSuccess) return GDN_ERR_CUDA;
    if (!mark()) return GDN_ERR_CUDA;
    return GDN_OK;
}

static gdn_status backward_impl(gdn_plan_t plan, const gdn_inputs *in, const void *dy, const gdn_grads *gr,
                                void *workspace, gdn_stream_t stream, void *const *events) {
    if (!plan || !in || !dy || !gr || !workspace) return GDN_ERR_INVALID_ARG;
    const gdn_config &c = plan->cfg;
    if (c.flags & GDN_FLAG_REVERSE) return GDN_ERR_UNSUPPORTED;
    const void *ptrs16[] = {in->q, in->k, in->v, in->z, dy, gr->dq, gr->dk, gr->dv, gr->dz};
    for (const void *q : ptrs16)
        if (!q || !aligned16(q)) return GDN_ERR_INVALID_ARG;
    const void *ptrs4[] = {in->g, in->b, in->conv_q, in->conv_k, in->conv_v, in->A_log, in->dt_bias, in->norm_w,
                           gr->dg, gr->db, gr->dconv_q, gr->dconv_k, gr->dconv_v, gr->dA_log, gr->ddt_bias,
                           gr->dnorm_w};
    for (const void *q : ptrs4)
        if (!q || (reinterpret_cast<uintptr_t>(q) & 3u)) return GDN_ERR_INVALID_ARG;
    const void *ptrsw[] = {in->conv_q, in->conv_k, in->conv_v};
    for (const void *q : ptrsw)
        if (!aligned16(q)) return GDN_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return GDN_ERR_INVALID_ARG;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != plan->device) return GDN_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    const int d = c.d_k;
    int *status = reinterpret_cast<int *>(ws + plan->b_status);
    if (cudaMemsetAsync(status, 0, sizeof(int), s) != cudaSuccess) return GDN_ERR_CUDA;
    auto F = [&](size_t off) { return reinterpret_cast<float *>(ws + off); };
    if (plan->tc_bwd) return backward_tc(plan, in, dy, gr, ws, s, events);

    PrepParams pp;
    memset(&pp, 0, sizeof(pp));
    pp.q = in->q; pp.k = in->k; pp.v = in->v;
    pp.tok_stride = plan->tok_stride;
    pp.g = in->g; pp.b = in->b;
    pp.conv_q = in->conv_q; pp.conv_k = in->conv_k; pp.conv_v = in->conv_v;
    pp.A_log = in->A_log; pp.dt_bias = in->dt_bias;
    pp.qh = F(plan->b_qh); pp.kh = F(plan->b_kh); pp.vh = F(plan->b_vh);
    pp.G = F(plan->b_G); pp.beta = F(plan->b_beta); pp.log_alpha = F(plan->b_la);
    pp.B = c.B; pp.T = c.T; pp.H = c.H; pp.d = d; pp.Tp = plan->Tp;
    pp.l2_eps = c.l2_eps;
    pp.q_scale = 1.0f / sqrtf(static_cast<float>(d));
    pp.status = status;
    pp.wait_limit_ns = kWaitLimitNs;
    pp.rev = 0;
    if (events && cudaEventRecord(reinterpret_cast<cudaEvent_t>(events[0]), s) != cudaSuccess) return GDN_ERR_CUDA;
    if (launch_prep(pp, in_type(c.in_dtype), false, s) != cudaSuccess) return GDN_ERR_CUDA;

    BwdParams bp;
    memset(&bp, 0, sizeof(bp));
    bp.groups = d / 8;
    bp.q = in->q; bp.k = in->k; bp.v = in->v; bp.z = in->z; bp.dy = dy;
    bp.tok_stride = plan->tok_stride;
    bp.g = in->g; bp.bg = in->b; bp.conv_q = in->conv_q; bp.conv_k = in->conv_k; bp.conv_v = in->conv_v;
    bp.A_log = in->A_log; bp.dt_bias = in->dt_bias; bp.norm_w = in->norm_w;
    bp.qh = F(plan->b_qh); bp.kh = F(plan->b_kh); bp.vh = F(plan->b_vh);
    bp.log_alpha = F(plan->b_la); bp.beta = F(plan->b_beta);
    bp.o = F(plan->b_o); bp.ckpt = F(plan->b_ckpt); bp.dO = F(plan->b_dO); bp.dvh = F(plan->b_dvh);
    bp.dq_part = F(plan->b_dqp); bp.dk_part = F(plan->b_dkp); bp.da_part = F(plan->b_dap); bp.db_part = F(plan->b_dbp);
    bp.dnw_part = F(plan->b_dnw); bp.dconv_part = F(plan->b_dconv); bp.dA_part = F(plan->b_dA);
    bp.ddt_part = F(plan->b_ddt);
    bp.dq = gr->dq; bp.dk = gr->dk; bp.dv = gr->dv; bp.dz = gr->dz; bp.dg = gr->dg; bp.db = gr->db;
    bp.dconv_q = gr->dconv_q; bp.dconv_k = gr->dconv_k; bp.dconv_v = gr->dconv_v;
    bp.dA_log = gr->dA_log; bp.ddt_bias = gr->ddt_bias; bp.dnorm_w = gr->dnorm_w;
    bp.B = c.B; bp.T = c.T; bp.H = c.H; bp.d = d; bp.Tp = plan->Tp;
    bp.l2_eps = c.l2_eps; bp.norm_eps = c.norm_eps; bp.q_scale = pp.q_scale;
    int n = 0;
    if (launch_backward(bp, in_type(c.in_dtype), in_type(c.out_dtype), s, &n, events ? events + 1 : nullptr) !=
        cudaSuccess)
        return GDN_ERR_CUDA;
    return GDN_OK;
}

gdn_status gdn_backward(gdn_plan_t plan, const gdn_inputs *in, const void *dy, const gdn_grads *gr, void *workspace,
                        gdn_stream_t stream) {
    return backward_impl(plan, in, dy, gr, workspace, stream, nullptr);
}

gdn_status gdn_backward_timed(gdn_plan_t plan, const gdn_inputs *in, const void *dy, const gdn_grads *gr,
                              void *workspace, gdn_stream_t stream, void *const *events, int n_events) {
    if (!plan || !events || n_events != gdn_backward_launches(plan) + 1) return GDN_ERR_INVALID_ARG;
    for (int i = 0; i < n_events; ++i)
        if (!events[i]) return GDN_ERR_INVALID_ARG;
    return backward_impl(plan, in, dy, gr, workspace, stream, events);
}

gdn_status gdn_get_device_status(gdn_plan_t plan, void *workspace, gdn_stream_t stream) {
    if (!plan || !workspace) return GDN_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int *status = reinterpret_cast<int *>(static_cast<uint8_t *>(workspace) + plan->off_status);
    int host = 0;
    if (cudaStreamSynchronize(s) != cudaSuccess) return GDN_ERR_CUDA;
    if (cudaMemcpy(&host, status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return GDN_ERR_CUDA;
    if (cudaMemset(status, 0, sizeof(int)) != cudaSuccess) return GDN_ERR_CUDA;
    if (host == kStatusTimeout) return GDN_ERR_TIMEOUT;
    if (host != kStatusOk) return GDN_ERR_DEVICE_CHECK;
    return GDN_OK;
}

}  // extern "C"
