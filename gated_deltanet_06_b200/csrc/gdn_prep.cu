// gdn_prep.cu -- K1 of the GDN forward: the per-token preparation the
// LinMorph page lists among the GDN module's parts ("Why learn the
// initialization?": short convolutions, normalization, decay terms, update
// gates), fused into one streaming pass:
//   q' k' v' = SiLU(causal depthwise conv4(x)),   q^ = q'/sqrt(|q'|^2+eps) / sqrt(d_k),
//   k^ = k'/sqrt(|k'|^2+eps),                      v^ = v',
//   log alpha = -exp(A_log) softplus(g + dt_bias), beta = sigmoid(b),
//   G = inclusive cumulative sum of log alpha inside each 128-token block.
// One CTA prepares 128 tokens of one (b, h); each thread owns 8 channels of a
// run of consecutive tokens, so the 3-token conv history is read once per run
// and every global access is a 16-byte vector.  Outputs are written head-major
// [B][H][Tp][d] (Tp = T rounded up to 128, padded rows zero, beta = 0,
// log alpha = 0) so that every 128-token block is one contiguous tile.
// For the reverse (anti-causal) scan the internal order is the reversed one:
// internal token t is input token T-1-t, so everything after this kernel
// runs unchanged, and the conv's history is the following input tokens.
#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

template <typename T>
struct In8;
template <>
struct In8<__nv_bfloat16> {
    static __device__ __forceinline__ void load(const __nv_bfloat16 *p, float (&f)[8]) {
        const uint4 u = *reinterpret_cast<const uint4 *>(p);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162 *>(&w[i]);
            float2 x = __bfloat1622float2(h);
            f[2 * i] = x.x;
            f[2 * i + 1] = x.y;
        }
    }
};
template <>
struct In8<__half> {
    static __device__ __forceinline__ void load(const __half *p, float (&f)[8]) {
        const uint4 u = *reinterpret_cast<const uint4 *>(p);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float2 x = unpack_half2(w[i]);
            f[2 * i] = x.x;
            f[2 * i + 1] = x.y;
        }
    }
};
template <>
struct In8<float> {
    static __device__ __forceinline__ void load(const float *p, float (&f)[8]) {
        const float4 a = reinterpret_cast<const float4 *>(p)[0];
        const float4 b = reinterpret_cast<const float4 *>(p)[1];
        f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
        f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
    }
};

template <typename OutT>
__device__ __forceinline__ void store8(OutT *p, const float (&f)[8]);
template <>
__device__ __forceinline__ void store8<__half>(__half *p, const float (&f)[8]) {
    uint4 u;
    u.x = pack_half2(f[0], f[1]);
    u.y = pack_half2(f[2], f[3]);
    u.z = pack_half2(f[4], f[5]);
    u.w = pack_half2(f[6], f[7]);
    *reinterpret_cast<uint4 *>(p) = u;
}
template <>
__device__ __forceinline__ void store8<float>(float *p, const float (&f)[8]) {
    reinterpret_cast<float4 *>(p)[0] = make_float4(f[0], f[1], f[2], f[3]);
    reinterpret_cast<float4 *>(p)[1] = make_float4(f[4], f[5], f[6], f[7]);
}

template <typename InT, typename OutT, int D>
__global__ void __launch_bounds__(256) gdn_prep_kernel(const PrepParams p) {
    constexpr int CPR = D / 8;      // 8-channel groups per token row
    constexpr int RG = 256 / CPR;   // token runs per CTA
    constexpr int RPT = kBlk / RG;  // tokens per run
    __shared__ float warp_tot[8];

    const int blk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int t0 = blk * kBlk;
    const int tid = threadIdx.x;
    const int cg = tid % CPR, rg = tid / CPR;
    const int c0 = cg * 8;
    const int rbeg = rg * RPT;
    const size_t bh = static_cast<size_t>(b) * p.H + h;

#pragma unroll 1
    for (int which = 0; which < 3; ++which) {
        const InT *x = static_cast<const InT *>(which == 0 ? p.q : (which == 1 ? p.k : p.v));
        const float *w = which == 0 ? p.conv_q : (which == 1 ? p.conv_k : p.conv_v);
        OutT *out = static_cast<OutT *>(which == 0 ? p.qh : (which == 1 ? p.kh : p.vh));

        float wt[8][4];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const float4 t = reinterpret_cast<const float4 *>(w)[static_cast<size_t>(h) * D + c0 + c];
            wt[c][0] = t.x; wt[c][1] = t.y; wt[c][2] = t.z; wt[c][3] = t.w;
        }
        float xin[RPT + 3][8];
#pragma unroll
        for (int i = 0; i < RPT + 3; ++i) {
            const int t = t0 + rbeg - 3 + i;
            if (t >= 0 && t < p.T) {
                const int ti = p.rev ? p.T - 1 - t : t;  // input token
                In8<InT>::load(x + (static_cast<size_t>(b) * p.T + ti) * p.tok_stride + static_cast<size_t>(h) * D + c0,
                               xin[i]);
            } else {
#pragma unroll
                for (int c = 0; c < 8; ++c) xin[i][c] = 0.0f;
            }
        }
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
            float u[8];
            float ss = 0.0f;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                float a = wt[c][0] * xin[r][c];
                a = fmaf(wt[c][1], xin[r + 1][c], a);
                a = fmaf(wt[c][2], xin[r + 2][c], a);
                a = fmaf(wt[c][3], xin[r + 3][c], a);
                u[c] = silu_f(a);
                ss = fmaf(u[c], u[c], ss);
            }
            if (which < 2) {
#pragma unroll
                for (int off = CPR / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
                float sc = 1.0f / sqrtf(ss + p.l2_eps);
                if (which == 0) sc *= p.q_scale;
#pragma unroll
                for (int c = 0; c < 8; ++c) u[c] *= sc;
            }
            const int t = t0 + rbeg + r;
            if (t >= p.T) {
#pragma unroll
                for (int c = 0; c < 8; ++c) u[c] = 0.0f;
            }
            store8<OutT>(out + (bh * p.Tp + t) * D + c0, u);
        }
    }

    // gates and the in-block cumulative log decay (threads 0..127, one token each)
    float la = 0.0f, be = 0.0f;
    const int t = t0 + tid;
    if (tid < kBlk && t < p.T) {
        const size_t gi = (static_cast<size_t>(b) * p.T + (p.rev ? p.T - 1 - t : t)) * p.H + h;
        const float xg = p.g[gi] + p.dt_bias[h];
        la = -expf(p.A_log[h]) * softplus_f(xg);
        be = 1.0f / (1.0f + expf(-p.b[gi]));
    }
    float cs = la;
    const int lane = tid & 31, wid = tid >> 5;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const float n = __shfl_up_sync(0xffffffffu, cs, off);
        if (lane >= off) cs += n;
    }
    if (lane == 31) warp_tot[wid] = cs;
    __syncthreads();
    if (tid < kBlk) {
        float pre = 0.0f;
        for (int i = 0; i < wid; ++i) pre += warp_tot[i];
        const size_t o = bh * p.Tp + t;
        p.G[o] = cs + pre;
        p.beta[o] = be;
        p.log_alpha[o] = la;
    }
}

// Tensor-path variant (16-bit inputs, d = 128), persistent: each CTA walks a
// contiguous range of 64-token tiles of the (b, h) sequences, with two
// stages of raw input in shared memory.  One thread issues the TMA loads of
// the next tile's three raw 67-token x 128-channel boxes (3 tokens of conv
// history; rows before t = 0 of the batch item and past T come back as zeros
// from the tensor map's out-of-bounds fill) while all 256 threads prepare
// the current one out of shared memory.  The conv weights of a head are
// staged once per change of head, which a contiguous range of tiles makes
// rare.  About 107 KB of shared memory: two CTAs per SM.  On this path the
// gates are evaluated by the chunk kernel, which needs them first.  For the
// reverse scan the box of internal tokens t0..t0+63 starts at input token
// T-64-t0 (its 3 extra rows are the following tokens, zero past T-1) and is
// read bottom-up: box row 66-k in place of row k.
constexpr int kPrepTok = 64;
constexpr int kRawRows = kPrepTok + 3;
constexpr uint32_t kRawTile = kRawRows * 256;          // bytes of one {128 ch, 67 tok} box (256-byte rows)
constexpr uint32_t kStage = 3 * kRawTile;              // q, k, v boxes of one tile
constexpr uint32_t kPrepW = 3 * 128 * 16;              // conv weights of q, k, v for one head (fp32)
constexpr uint32_t kPrepSmem = 2 * kStage + kPrepW + 64 + 128;
static_assert(kRawTile % 128 == 0, "TMA destinations stay 128-byte aligned");

template <typename InT>
__global__ void __launch_bounds__(256, 2)
    gdn_prep_tma_kernel(const PrepParams p, const __grid_constant__ CUtensorMap tmq,
                        const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv) {
    constexpr int D = 128, CPR = 16, RPT = 4;
    extern __shared__ __align__(128) uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    float4 *sW = reinterpret_cast<float4 *>(sm + 2 * kStage);  // [3][128] taps
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + 2 * kStage + kPrepW);  // one per stage
    __shared__ AbortState ab;

    const int nparts = p.Tp / kPrepTok;
    const int ntiles = nparts * p.H * p.B;  // tile L = (b * H + h) * nparts + part
    const int per = (ntiles + gridDim.x - 1) / gridDim.x;
    const int first = blockIdx.x * per, last = min(first + per, ntiles);
    const int tid = threadIdx.x;
    // debug: the CTA's output rows (tiles first..last-1 of kPrepTok rows) inside q^, k^, v^
    if (p.debug) {
        const bool ok = p.Tp % kPrepTok == 0 &&
                        debug_in_bounds(1, static_cast<size_t>(first) * kPrepTok,
                                        static_cast<size_t>(max(last - first, 0)) * kPrepTok,
                                        static_cast<size_t>(p.B) * p.H * p.Tp, p.status);
        if (!ok) {
            atomicCAS(p.status, kStatusOk, kStatusCheck);
            return;
        }
    }
    if (tid == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        ab.flag = 0;
        fence_mbar_init();
    }
    pdl_launch_dependents();
    __syncthreads();
    auto issue = [&](int n, int L) {  // thread 0: the raw boxes of tile L into stage n & 1
        const int part = L % nparts, bh = L / nparts;
        const int h = bh % p.H, b = bh / p.H;
        uint8_t *dst = sm + (n & 1) * kStage;
        mbar_arrive_expect_tx(&bar[n & 1], kStage);
        const CUtensorMap *maps[3] = {&tmq, &tmk, &tmv};
        for (int w = 0; w < 3; ++w)
            asm volatile(
                "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(
                    smem_u32(dst + w * kRawTile)),
                "l"(maps[w]), "r"(smem_u32(&bar[n & 1])), "r"(h * D),
                "r"(p.rev ? p.T - kPrepTok - part * kPrepTok : part * kPrepTok - 3), "r"(b)
                : "memory");
    };
    if (tid == 0 && first < last) issue(0, first);

    const int cg = tid % CPR, rg = tid / CPR;
    const int c0 = cg * 8;
    const int rbeg = rg * RPT;
    const uint32_t coff = cg * 16;
    // box row of window row k (k = 0..66; k = r + 3 is internal token t0 + r)
    const int rsign = p.rev ? -256 : 256, rzero = p.rev ? 66 * 256 : 0;
    int cur_h = -1;
    for (int L = first, n = 0; L < last; ++L, ++n) {
        if (tid == 0 && L + 1 < last) issue(n + 1, L + 1);  // stage (n+1)&1 was released at the end of tile n-1
        const int part = L % nparts, bh = L / nparts;
        const int h = bh % p.H;
        const int t0 = part * kPrepTok;  // first token of this tile
        if (h != cur_h) {
            // conv taps of this head, laid out [tensor][channel-in-group][group] so that the 16
            // threads of a token row read 16 consecutive float4
            for (int i = tid; i < 3 * 128; i += 256) {
                const int which = i >> 7, ch = i & 127;
                const float *w = which == 0 ? p.conv_q : (which == 1 ? p.conv_k : p.conv_v);
                sW[which * 128 + (ch & 7) * 16 + (ch >> 3)] =
                    reinterpret_cast<const float4 *>(w)[static_cast<size_t>(h) * D + ch];
            }
            cur_h = h;
        }
        const bool ok = mbar_wait(&bar[n & 1], (n >> 1) & 1, &ab, p.status, p.wait_limit_ns);
        if (!__syncthreads_and(ok)) {  // (also publishes the taps)
            // boxes still in flight (this tile's, and the next tile's if issued) land before the
            // CTA's shared memory goes away (bounded waits that ignore the abort flag)
            if (tid == 0) {
                mbar_wait_drain(&bar[n & 1], (n >> 1) & 1, p.wait_limit_ns);
                if (L + 1 < last) mbar_wait_drain(&bar[(n + 1) & 1], ((n + 1) >> 1) & 1, p.wait_limit_ns);
            }
            return;
        }
        if (tid == 0 && n == 0) GDN_TRACE_AT(0);
        const uint8_t *stage = sm + (n & 1) * kStage;
#pragma unroll 1
        for (int which = 0; which < 3; ++which) {
            __half *out = static_cast<__half *>(which == 0 ? p.qh : (which == 1 ? p.kh : p.vh));
            const uint8_t *tile = stage + which * kRawTile + coff;
            float4 wt[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) wt[c] = sW[which * 128 + c * 16 + cg];
            float win[4][8];
#pragma unroll
            for (int i = 0; i < 3; ++i)
                In8<InT>::load(reinterpret_cast<const InT *>(tile + rzero + (rbeg + i) * rsign), win[i]);
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                In8<InT>::load(reinterpret_cast<const InT *>(tile + rzero + (rbeg + r + 3) * rsign), win[(r + 3) & 3]);
                float u[8];
                float ss = 0.0f;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    float a = wt[c].x * win[r & 3][c];
                    a = fmaf(wt[c].y, win[(r + 1) & 3][c], a);
                    a = fmaf(wt[c].z, win[(r + 2) & 3][c], a);
                    a = fmaf(wt[c].w, win[(r + 3) & 3][c], a);
                    u[c] = silu_tc(a);
                    ss = fmaf(u[c], u[c], ss);
                }
                if (which < 2) {
#pragma unroll
                    for (int off = CPR / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
                    float sc = rsqrtf(ss + p.l2_eps);
                    if (which == 0) sc *= p.q_scale;
#pragma unroll
                    for (int c = 0; c < 8; ++c) u[c] *= sc;
                }
                const int t = t0 + rbeg + r;
                if (t >= p.T) {
#pragma unroll
                    for (int c = 0; c < 8; ++c) u[c] = 0.0f;
                }
                store8<__half>(out + (static_cast<size_t>(bh) * p.Tp + t) * D + c0, u);
            }
        }
        __syncthreads();  // every read of this stage and of the taps is done
    }
}

template <typename InT, typename OutT>
cudaError_t launch_typed(const PrepParams &p, cudaStream_t s) {
    dim3 grid(p.Tp / kBlk, p.H, p.B);
    if (p.d == 128)
        gdn_prep_kernel<InT, OutT, 128><<<grid, 256, 0, s>>>(p);
    else
        gdn_prep_kernel<InT, OutT, 64><<<grid, 256, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prep_tma(const PrepParams &p, InType in, const CUtensorMap &tmq, const CUtensorMap &tmk,
                            const CUtensorMap &tmv, cudaStream_t s) {
    static SmemOnce once_bf, once_h;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return cudaErrorInvalidDevice;
    const long long ntiles = static_cast<long long>(p.Tp / kPrepTok) * p.H * p.B;
    dim3 grid(static_cast<unsigned>(ntiles < 2LL * sms ? ntiles : 2LL * sms));
    if (in == InType::BF16) {
        cudaError_t e = raise_smem_once(once_bf, gdn_prep_tma_kernel<__nv_bfloat16>, static_cast<int>(kPrepSmem));
        if (e != cudaSuccess) return e;
        gdn_prep_tma_kernel<__nv_bfloat16><<<grid, 256, kPrepSmem, s>>>(p, tmq, tmk, tmv);
    } else {
        cudaError_t e = raise_smem_once(once_h, gdn_prep_tma_kernel<__half>, static_cast<int>(kPrepSmem));
        if (e != cudaSuccess) return e;
        gdn_prep_tma_kernel<__half><<<grid, 256, kPrepSmem, s>>>(p, tmq, tmk, tmv);
    }
    return cudaGetLastError();
}

cudaError_t launch_prep(const PrepParams &p, InType in, bool out_f16, cudaStream_t s) {
    if (out_f16) {
        if (in == InType::BF16) return launch_typed<__nv_bfloat16, __half>(p, s);
        if (in == InType::F16) return launch_typed<__half, __half>(p, s);
        return launch_typed<float, __half>(p, s);
    }
    if (in == InType::BF16) return launch_typed<__nv_bfloat16, float>(p, s);
    if (in == InType::F16) return launch_typed<__half, float>(p, s);
    return launch_typed<float, float>(p, s);
}

}  // namespace gdn

GDN_TRACE_EXPORT(prep)
