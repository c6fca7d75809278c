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

