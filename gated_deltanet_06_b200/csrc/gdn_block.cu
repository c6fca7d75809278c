// gdn_block.cu -- the C ABI of the GDN layer with its projections
// (gdn_block_*): the input projection with the fused conv / SiLU / L2
// epilogue (gdn_proj.cu), the tensor path's UT transform and segment-parallel
// scan (gdn_chunk.cu, gdn_scan.cu), and the output projection.  No device
// memory is allocated here; every buffer is the caller's.
#include <math.h>
#include <string.h>

#include <new>

#include "gdn.h"
#include "gdn_common.cuh"
#include "gdn_internal.h"

using namespace gdn;

struct gdn_block_plan_s {
    gdn_block_config cfg;
    gdn_plan_t core;     // the tensor-path plan of the GDN core (fp16 y)
    PlanLayout lay;      // its workspace layout (at the start of the block workspace)
    int device;
    int M, Hd, Nin;      // token rows, H*d, rows of W_in
    size_t off_z, off_g, off_b, off_y, off_wo, ws_bytes;
};

namespace {

constexpr unsigned long long kWaitLimitNs = 2000ull * 1000 * 1000;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// [rows][K] 16-bit row-major (K-major GEMM operand), {64, box_rows} boxes with the 128-byte
// swizzle; rows past the end (and, for loads, negative rows) read as zero.
bool make_kmajor_map(CUtensorMap *m, const void *base, unsigned long long rows, unsigned long long K,
                     unsigned box_rows, bool f16 = false) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {K, rows};
    const cuuint64_t strides[1] = {K * 2};
    const cuuint32_t box[2] = {64, box_rows};
    const cuuint32_t es[2] = {1, 1};
    return enc(m, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
               const_cast<void *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

gdn_status block_forward(gdn_block_plan_t plan, const gdn_block_inputs *in, void *out, void *workspace,
                         gdn_stream_t stream, void *const *events) {
    if (!plan || !in || !out || !workspace) return GDN_ERR_INVALID_ARG;
    const gdn_block_config &c = plan->cfg;
    const void *p16[] = {in->x, in->w_in, in->w_out, out, in->conv_q, in->conv_k, in->conv_v};
    for (const void *q : p16)
        if (!q || !aligned16(q)) return GDN_ERR_INVALID_ARG;
    const void *p4[] = {in->A_log, in->dt_bias, in->norm_w};
    for (const void *q : p4)
        if (!q || (reinterpret_cast<uintptr_t>(q) & 3u)) return GDN_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return GDN_ERR_INVALID_ARG;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != plan->device) return GDN_ERR_INVALID_ARG;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    const PlanLayout &L = plan->lay;
    int *status = reinterpret_cast<int *>(ws + L.off_status);
    __half *z = reinterpret_cast<__half *>(ws + plan->off_z);
    float *g = reinterpret_cast<float *>(ws + plan->off_g);
    float *b = reinterpret_cast<float *>(ws + plan->off_b);
    void *y = ws + plan->off_y;
    void *wo16 = ws + plan->off_wo;
    int ev = 0;
    auto mark = [&]() -> bool {
        if (!events) return true;
        return cudaEventRecord(reinterpret_cast<cudaEvent_t>(events[ev++]), s) == cudaSuccess;
    };

    CUtensorMap tmX, tmWin, tmY, tmWout;
    if (!make_kmajor_map(&tmX, in->x, plan->M, c.D, 128) || !make_kmajor_map(&tmWin, in->w_in, plan->Nin, c.D, 256) ||
        !make_kmajor_map(&tmY, y, plan->M, plan->Hd, 128, true) ||
        !make_kmajor_map(&tmWout, wo16, c.D, plan->Hd, 256, true))
        return GDN_ERR_CUDA;

    if (!mark()) return GDN_ERR_CUDA;
    if (cudaMemsetAsync(status, 0, sizeof(int), s) != cudaSuccess) return GDN_ERR_CUDA;
    // the output projection runs on fp16 operands: y leaves the scan in fp16 (3 more mantissa bits
    // than bf16), and W_out is copied to fp16 to match it
    if (launch_bf16_to_f16(in->w_out, wo16, static_cast<size_t>(c.D) * plan->Hd, s) != cudaSuccess)
        return GDN_ERR_CUDA;
    if (L.Tp > L.T) {  // the operand rows past T of every (b, h) are zero, as the UT transform expects
        const size_t row = kD * sizeof(__half);
        const size_t offs[3] = {L.off_qh, L.off_kh, L.off_vh};
        for (size_t o : offs)
            if (cudaMemset2DAsync(ws + o + static_cast<size_t>(L.T) * row, static_cast<size_t>(L.Tp) * row, 0,
                                  static_cast<size_t>(L.Tp - L.T) * row, static_cast<size_t>(L.B) * L.H, s) != cudaSuccess)
                return GDN_ERR_CUDA;
    }

    ProjParams pi;
    memset(&pi, 0, sizeof(pi));
    pi.M = plan->M; pi.N = plan->Nin; pi.K = c.D;
    pi.m_step = proj_m_step(0);
    pi.m_tiles = (plan->M + pi.m_step - 1) / pi.m_step;
    pi.n_tiles = 2 * c.H + 1;  // two heads of q, k, v or z per tile, then the g | b tile
    pi.B = c.B; pi.T = c.T; pi.H = c.H; pi.Tp = L.Tp;
    pi.conv_q = in->conv_q; pi.conv_k = in->conv_k; pi.conv_v = in->conv_v;
    pi.qh = reinterpret_cast<__half *>(ws + L.off_qh);
    pi.kh = reinterpret_cast<__half *>(ws + L.off_kh);
    pi.vh = reinterpret_cast<__half *>(ws + L.off_vh);
    pi.z = z; pi.g = g; pi.b = b;
    pi.l2_eps = c.l2_eps;
    pi.q_scale = 1.0f / sqrtf(static_cast<float>(c.d));
    pi.debug = (c.flags & GDN_FLAG_DEBUG_CHECKS) ? 1 : 0;
    pi.status = status;
    pi.wait_limit_ns = kWaitLimitNs;
    if (!mark() || launch_proj(pi, 0, tmX, tmWin, s, false) != cudaSuccess) return GDN_ERR_CUDA;

    const int st = run_tensor_core(plan->core, g, b, in->A_log, in->dt_bias, in->norm_w, z, InType::F16, plan->Hd, y,
                                   workspace, s, events == nullptr, events, &ev, nullptr, nullptr);
    if (st != GDN_OK) return static_cast<gdn_status>(st);

    ProjParams po;
    memset(&po, 0, sizeof(po));
    po.M = plan->M; po.N = c.D; po.K = plan->Hd;
    po.m_step = proj_m_step(1);
    po.m_tiles = (plan->M + po.m_step - 1) / po.m_step;
    po.n_tiles = (c.D + proj_n_tile() - 1) / proj_n_tile();
    po.out = out;
    po.out_kind = c.out_dtype == GDN_DTYPE_F32 ? 1 : 0;
    po.f16 = 1;
    po.debug = pi.debug;
    po.status = status;
    po.wait_limit_ns = kWaitLimitNs;
    if (!mark() || launch_proj(po, 1, tmY, tmWout, s, events == nullptr) != cudaSuccess) return GDN_ERR_CUDA;
    if (!mark()) return GDN_ERR_CUDA;
    return GDN_OK;
}

}  // namespace

extern "C" {

gdn_status gdn_block_plan(const gdn_block_config *cfg, gdn_block_plan_t *out, size_t *workspace_bytes) {
    if (!cfg || !out || !workspace_bytes) return GDN_ERR_INVALID_ARG;
    *out = nullptr;
    const gdn_block_config c = *cfg;
    if (c.B < 1 || c.T < 1 || c.H < 1 || c.d < 1 || c.D < 1) return GDN_ERR_INVALID_ARG;
    if (c.d != 128 || (c.H & 1) || c.D % 64 != 0 || c.H > 64) return GDN_ERR_UNSUPPORTED;
    if (c.out_dtype != GDN_DTYPE_BF16 && c.out_dtype != GDN_DTYPE_F32) return GDN_ERR_UNSUPPORTED;
    if (c.flags & ~GDN_FLAG_DEBUG_CHECKS) return GDN_ERR_UNSUPPORTED;
    const long long M = static_cast<long long>(c.B) * c.T;
    if (M >= (1ll << 31) - 256) return GDN_ERR_UNSUPPORTED;

    gdn_config core;
    memset(&core, 0, sizeof(core));
    core.B = c.B; core.T = c.T; core.H = c.H; core.d_k = core.d_v = c.d;
    core.in_dtype = GDN_DTYPE_BF16; core.out_dtype = GDN_DTYPE_F16;
    core.conv_size = 4; core.chunk = 64;
    core.l2_eps = c.l2_eps; core.norm_eps = c.norm_eps;
    core.flags = c.flags & GDN_FLAG_DEBUG_CHECKS;
    gdn_plan_t cp = nullptr;
    size_t cws = 0;
    const gdn_status st = gdn_plan(&core, &cp, &cws);
    if (st != GDN_OK) return st;

    gdn_block_plan_s *p = new (std::nothrow) gdn_block_plan_s;
    if (!p) {
        gdn_destroy(cp);
        return GDN_ERR_INVALID_ARG;
    }
    memset(p, 0, sizeof(*p));
    p->cfg = c;
    p->core = cp;
    if (!plan_layout(cp, &p->lay)) {
        gdn_destroy(cp);
        delete p;
        return GDN_ERR_UNSUPPORTED;
    }
    cudaGetDevice(&p->device);
    p->M = static_cast<int>(M);
    p->Hd = c.H * c.d;
    p->Nin = 4 * p->Hd + 2 * c.H;
    const size_t A = 1024;
    size_t off = align_up(p->lay.ws_bytes, A);
    p->off_z = off; off = align_up(off + static_cast<size_t>(M) * p->Hd * 2, A);
    p->off_g = off; off = align_up(off + static_cast<size_t>(M) * c.H * 4, A);
    p->off_b = off; off = align_up(off + static_cast<size_t>(M) * c.H * 4, A);
    p->off_y = off; off = align_up(off + static_cast<size_t>(M) * p->Hd * 2, A);
    p->off_wo = off; off = align_up(off + static_cast<size_t>(c.D) * p->Hd * 2, A);
    p->ws_bytes = off;
    *out = p;
    *workspace_bytes = off;
    return GDN_OK;
}

gdn_status gdn_block_forward(gdn_block_plan_t plan, const gdn_block_inputs *in, void *out, void *workspace,
                             gdn_stream_t stream) {
    return block_forward(plan, in, out, workspace, stream, nullptr);
}

gdn_status gdn_block_forward_timed(gdn_block_plan_t plan, const gdn_block_inputs *in, void *out, void *workspace,
                                   gdn_stream_t stream, void *const *events, int n_events) {
    if (!plan || !events || n_events != gdn_block_launches(plan) + 1) return GDN_ERR_INVALID_ARG;
    for (int i = 0; i < n_events; ++i)
        if (!events[i]) return GDN_ERR_INVALID_ARG;
    return block_forward(plan, in, out, workspace, stream, events);
}

int gdn_block_launches(gdn_block_plan_t plan) { return plan ? 3 + tensor_core_launches(plan->core) : 0; }

gdn_status gdn_block_device_status(gdn_block_plan_t plan, void *workspace, gdn_stream_t stream) {
    if (!plan) return GDN_ERR_INVALID_ARG;
    return gdn_get_device_status(plan->core, workspace, stream);
}

gdn_status gdn_block_destroy(gdn_block_plan_t plan) {
    if (!plan) return GDN_OK;
    gdn_destroy(plan->core);
    delete plan;
    return GDN_OK;
}

}  // extern "C"
