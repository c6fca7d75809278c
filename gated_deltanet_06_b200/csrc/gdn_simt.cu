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

// Thread i owns row i of S (d_k values in registers).  Per token:
//   u = S_i . k;  S_i <- alpha (S_i - beta u k) + beta v_i k;  o_i = S_i . q^
// (q^ already carries 1/sqrt(d_k)).  Rows of S evolve independently, so no
// cross-thread reduction is needed; k, q, v tiles of 16 tokens are staged in
// shared memory.
template <int D>
__global__ void __launch_bounds__(D) gdn_recurrence_kernel(const RecurParams p) {
    constexpr int TT = 16;
    __shared__ float sk[TT][D], sq[TT][D], sv[TT][D], sa[TT], sb[TT];
    const int h = blockIdx.x, b = blockIdx.y, i = threadIdx.x;
    const size_t bh = static_cast<size_t>(b) * p.H + h;
    float S[D];  // row i of the state (d_v index i, d_k index j)
    const float *s0 = p.s0 ? p.s0 + (bh * D + i) * D : nullptr;
#pragma unroll
    for (int j = 0; j < D; ++j) S[j] = s0 ? s0[j] : 0.0f;
    for (int t0 = 0; t0 < p.T; t0 += TT) {
        __syncthreads();
#pragma unroll 4
        for (int tok = 0; tok < TT; ++tok) {
            const size_t rrow = (bh * p.Tp + t0 + tok) * D + i;
            sk[tok][i] = p.kh[rrow];
            sq[tok][i] = p.qh[rrow];
            sv[tok][i] = p.vh[rrow];
        }
        if (i < TT) {
            sa[i] = expf(p.log_alpha[bh * p.Tp + t0 + i]);
            sb[i] = p.beta[bh * p.Tp + t0 + i];
        }
        __syncthreads();
        const int n = min(TT, p.T - t0);
        for (int tok = 0; tok < n; ++tok) {
            float u = 0.0f;
#pragma unroll
            for (int j = 0; j < D; ++j) u = fmaf(S[j], sk[tok][j], u);
            const float a = sa[tok], be = sb[tok];
            const float c1 = be * u, c2 = be * sv[tok][i];
            float o = 0.0f;
#pragma unroll
            for (int j = 0; j < D; ++j) {
                const float kj = sk[tok][j];
                S[j] = fmaf(a, fmaf(-c1, kj, S[j]), c2 * kj);
                o = fmaf(S[j], sq[tok][j], o);
            }
            const int to = p.rev ? p.T - 1 - (t0 + tok) : t0 + tok;  // input token order
            p.o[((static_cast<size_t>(b) * p.T + to) * p.H + h) * D + i] = o;
        }
    }
    if (p.s_end) {
        float *se = p.s_end + (bh * D + i) * D;
#pragma unroll
        for (int j = 0; j < D; ++j) se[j] = S[j];
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
        gdn_recurrence_kernel<128><<<grid, 128, 0, s>>>(p);
    else
        gdn_recurrence_kernel<64><<<grid, 64, 0, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_output(const OutParams &p, InType zt, InType yt, cudaStream_t s) {
    if (zt == InType::BF16) return launch_out_z<__nv_bfloat16>(p, yt, s);
    if (zt == InType::F16) return launch_out_z<__half>(p, yt, s);
    return launch_out_z<float>(p, yt, s);
}

}  // namespace gdn
