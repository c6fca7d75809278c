// gdn_simt.cu -- the CUDA-core kernels of the GDN forward:
//  * the token-sequential fp32 recurrence of the gated delta rule (reference
//    [57] on the VMonarch page), used for fp32 inputs, whose tolerance rules
//    out fp16/bf16/tf32 tensor-core operands, and for d = 64;
//  * the output step the LinMorph page counts among the module's
//    normalization parameters: y = o / sqrt(mean(o^2) + eps) * w * SiLU(z).
#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

// Four threads own row i of S, a quarter of its d_k values each, in registers.  Per token:
//   u = S_i . k;  S_i <- alpha (S_i - beta u k) + beta v_i k;  o_i = S_i . q^
// (q^ already carries 1/sqrt(d_k)).  Rows of S evolve independently; the two dot products of a
// row are split over its four threads in four short partial sums each and added with two
// shuffles, so that a token costs a few dependent steps rather than a d_k-long chain.  k, q, v
// tiles of 16 tokens (8 at d_k = 128) are double-buffered in shared memory, the next tile's global loads in
// flight in registers while the current one is processed.
template <int D>
__global__ void __launch_bounds__(4 * D) gdn_recurrence_kernel(const RecurParams p) {
    constexpr int TT = D == 128 ? 8 : 16, Q = D / 4;  // tokens per staged tile (48 KB of static smem); columns per thread
    __shared__ __align__(16) float sk[2][TT][D];
    __shared__ __align__(16) float sq[2][TT][D];
    __shared__ float sv[2][TT][D], sa[2][TT], sb[2][TT];
    const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
    const int i = tid >> 2, part = tid & 3, j0 = part * Q;  // row of S; this thread's columns j0 .. j0+Q-1
    const size_t bh = static_cast<size_t>(b) * p.H + h;
    float S[Q];
    const float *s0 = p.s0 ? p.s0 + (bh * D + i) * D + j0 : nullptr;
#pragma unroll
    for (int j = 0; j < Q; ++j) S[j] = s0 ? s0[j] : 0.0f;
    // this thread's share of a tile: TT / 4 elements of each of k, q, v (and one gate pair)
    constexpr int PER = TT * D / (4 * D);
    float rk[PER], rq[PER], rv[PER], ra = 0.0f, rb = 0.0f;
    auto fetch = [&](int t0) {  // global -> registers
#pragma unroll
        for (int e = 0; e < PER; ++e) {
            const int idx = tid + e * 4 * D, tok = idx / D, c = idx - tok * D;
            const size_t rrow = (bh * p.Tp + t0 + tok) * D + c;
            rk[e] = p.kh[rrow];
            rq[e] = p.qh[rrow];
            rv[e] = p.vh[rrow];
        }
        if (tid < TT) {
            ra = expf(p.log_alpha[bh * p.Tp + t0 + tid]);
            rb = p.beta[bh * p.Tp + t0 + tid];
        }
    };
    auto stage = [&](int buf) {  // registers -> shared memory
#pragma unroll
        for (int e = 0; e < PER; ++e) {
            const int idx = tid + e * 4 * D, tok = idx / D, c = idx - tok * D;
            sk[buf][tok][c] = rk[e];
            sq[buf][tok][c] = rq[e];
            sv[buf][tok][c] = rv[e];
        }
        if (tid < TT) {
            sa[buf][tid] = ra;
            sb[buf][tid] = rb;
        }
    };
    fetch(0);
    stage(0);
    __syncthreads();
    for (int t0 = 0, buf = 0; t0 < p.T; t0 += TT, buf ^= 1) {
        const bool more = t0 + TT < p.T;
        if (more) fetch(t0 + TT);  // the next tile's loads are in flight while this one is processed
        const int n = min(TT, p.T - t0);
        for (int tok = 0; tok < n; ++tok) {
            float k[Q], q[Q];
#pragma unroll
            for (int j = 0; j < Q; j += 4) {
                const float4 k4 = *reinterpret_cast<const float4 *>(&sk[buf][tok][j0 + j]);
                const float4 q4 = *reinterpret_cast<const float4 *>(&sq[buf][tok][j0 + j]);
                k[j] = k4.x; k[j + 1] = k4.y; k[j + 2] = k4.z; k[j + 3] = k4.w;
                q[j] = q4.x; q[j + 1] = q4.y; q[j + 2] = q4.z; q[j + 3] = q4.w;
            }
            float u4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
            for (int j = 0; j < Q; ++j) u4[j & 3] = fmaf(S[j], k[j], u4[j & 3]);
            float u = (u4[0] + u4[1]) + (u4[2] + u4[3]);
            u += __shfl_xor_sync(0xffffffffu, u, 1);
            u += __shfl_xor_sync(0xffffffffu, u, 2);
            const float a = sa[buf][tok], be = sb[buf][tok];
            const float c1 = be * u, c2 = be * sv[buf][tok][i];
            float o4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
            for (int j = 0; j < Q; ++j) {
                S[j] = fmaf(a, fmaf(-c1, k[j], S[j]), c2 * k[j]);
                o4[j & 3] = fmaf(S[j], q[j], o4[j & 3]);
            }
            float o = (o4[0] + o4[1]) + (o4[2] + o4[3]);
            o += __shfl_xor_sync(0xffffffffu, o, 1);
            o += __shfl_xor_sync(0xffffffffu, o, 2);
            const int to = p.rev ? p.T - 1 - (t0 + tok) : t0 + tok;  // input token order
            if (part == 0) p.o[((static_cast<size_t>(b) * p.T + to) * p.H + h) * D + i] = o;
        }
        if (more) stage(buf ^ 1);  // the other buffer's last readers finished before the previous barrier
        __syncthreads();
    }
    if (p.s_end) {
        float *se = p.s_end + (bh * D + i) * D + j0;
#pragma unroll
        for (int j = 0; j < Q; ++j) se[j] = S[j];
    }
}

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }
template <>
__device__ __forceinline__ float to_f<__half>(__half x) { return __half2float(x); }

template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }
template <>
__device__ __forceinline__ __half from_f<__half>(float x) { return __float2half_rn(x); }

// One warp per (b, t, h) row of d_v values.
template <typename ZT, typename YT, int DV>
__global__ void __launch_bounds__(256) gdn_output_kernel(const OutParams p) {
    constexpr int PER = DV / 32;
    const int lane = threadIdx.x & 31;
    const long long nrows = static_cast<long long>(p.B) * p.T * p.H;
    const long long wpb = blockDim.x / 32;
    float w[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) w[e] = p.norm_w[lane * PER + e];
    const ZT *z = static_cast<const ZT *>(p.z);
    YT *y = static_cast<YT *>(p.y);
    for (long long row = blockIdx.x * wpb + threadIdx.x / 32; row < nrows; row += gridDim.x * wpb) {
        const float *o = p.o + row * DV + lane * PER;
        float ov[PER];
        float ss = 0.0f;
#pragma unroll
        for (int e = 0; e < PER; ++e) {
            ov[e] = o[e];
            ss = fmaf(ov[e], ov[e], ss);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        const float rn = 1.0f / sqrtf(ss / DV + p.eps);
        const long long tok = row / p.H, hh = row % p.H;
        const ZT *zr = z + tok * p.tok_stride + hh * DV + lane * PER;
        YT *yr = y + row * DV + lane * PER;
#pragma unroll
        for (int e = 0; e < PER; ++e) {
            const float v = ov[e] * rn * w[e] * silu_f(to_f<ZT>(zr[e]));
            if (p.debug && !isfinite(v)) atomicCAS(p.status, kStatusOk, kStatusCheck);
            yr[e] = from_f<YT>(v);
        }
    }
}

template <typename ZT, typename YT>
cudaError_t launch_out_typed(const OutParams &p, cudaStream_t s) {
    const long long nrows = static_cast<long long>(p.B) * p.T * p.H;
    long long blocks = (nrows + 7) / 8;
    if (blocks > 148 * 16) blocks = 148 * 16;
    if (p.dv == 128)
        gdn_output_kernel<ZT, YT, 128><<<static_cast<unsigned>(blocks), 256, 0, s>>>(p);
    else
        gdn_output_kernel<ZT, YT, 64><<<static_cast<unsigned>(blocks), 256, 0, s>>>(p);
    return cudaGetLastError();
}

template <typename ZT>
cudaError_t launch_out_z(const OutParams &p, InType yt, cudaStream_t s) {
    if (yt == InType::BF16) return launch_out_typed<ZT, __nv_bfloat16>(p, s);
    if (yt == InType::F16) return launch_out_typed<ZT, __half>(p, s);
    return launch_out_typed<ZT, float>(p, s);
}

}  // namespace

cudaError_t launch_recurrence(const RecurParams &p, cudaStream_t s) {
    dim3 grid(p.H, p.B);
    if (p.d == 128)
        gdn_recurrence_kernel<128><<<grid, 512, 0, s>>>(p);
    else
        gdn_recurrence_kernel<64><<<grid, 256, 0, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_output(const OutParams &p, InType zt, InType yt, cudaStream_t s) {
    if (zt == InType::BF16) return launch_out_z<__nv_bfloat16>(p, yt, s);
    if (zt == InType::F16) return launch_out_z<__half>(p, yt, s);
    return launch_out_z<float>(p, yt, s);
}

}  // namespace gdn
