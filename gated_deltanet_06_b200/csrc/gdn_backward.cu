// gdn_backward.cu -- the gradient of the GDN forward (the gated delta rule of
// reference [57] on the VMonarch page, with the LinMorph page's short
// convolutions, normalizations, decay terms and update gates) with respect to
// every input and parameter, in fp32 on CUDA cores.
//
// The recurrence, rearranged: u_t = S_{t-1} k^_t, delta_t = beta_t (v^_t -
// alpha_t u_t), S_t = alpha_t S_{t-1} + delta_t k^_t^T, o_t = S_t q^_t.  Row i
// of S (a d_v index) only ever meets row i of S, forwards and backwards: with
// D_t = dL/dS_t,
//   D_t += do_t q^_t^T;  ddelta = D_t k^_t;  du = -alpha beta ddelta;
//   D_{t-1} = alpha D_t + du k^_t^T,
// so the state and its gradient split into groups of R = 8 rows, one CTA per
// (group, head).  What does couple the rows are the outputs
//   dq^_t = S_t^T do_t,  dk^_t = D_t^T delta_t + S_{t-1}^T du,
//   dalpha_t = <D_t, S_{t-1}> - beta u.ddelta,  dbeta_t = ddelta.(v^ - alpha u),
// sums over rows that feed nothing back: each CTA writes its group's partial
// sums, and the token kernel adds the groups.  Kernels, in order:
//   prep (the forward's fp32 prep, recomputed) -> gdn_bwd_fwd_rows (o and a
//   checkpoint of S every C = 8 tokens) -> gdn_bwd_out (RMSNorm and SiLU(z)
//   gate backwards: do, dz, norm-weight partials) -> gdn_bwd_core (per chunk
//   of C tokens, last to first: states recomputed from the checkpoint into
//   shared memory, the gradient run backwards, the row sums taken from shared
//   memory) -> gdn_bwd_tokens (group sums, L2-norm, SiLU and conv backwards,
//   gates) -> gdn_bwd_params_split (sums over tokens of the parameter gradients).
// The output-step, per-token and parameter kernels also serve the tensor-core
// backward (gdn_bwd_tc.cu), which hands them dO in fp16, whole per-token
// gradients of q^ k^ v^ and d log alpha; its per-token step is
// gdn_bwd_tokens_rows (one warp per token row).
#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int kR = 8;     // rows of S per CTA
constexpr int kC = 8;     // tokens per checkpoint chunk
constexpr int kTile = 64; // tokens per CTA of the token kernel
constexpr int kBT = 256;  // threads per CTA of the row kernels: one warp per row of S

template <typename T>
__device__ __forceinline__ float ldf(const T *p);
template <>
__device__ __forceinline__ float ldf<float>(const float *p) { return *p; }
template <>
__device__ __forceinline__ float ldf<__nv_bfloat16>(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
template <>
__device__ __forceinline__ float ldf<__half>(const __half *p) { return __half2float(*p); }

__device__ __forceinline__ float sigm(float x) { return 1.0f / (1.0f + expf(-x)); }
// d SiLU(a) / da
__device__ __forceinline__ float dsilu(float a) {
    const float s = sigm(a);
    return s * (1.0f + a * (1.0f - s));
}
// sum over the 32 lanes of a warp (one row of S)
__device__ __forceinline__ float rowsum(float x) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
}

// ------------------------------------------------------------ forward rows
// One CTA per (group of kR rows, h, b), kBT threads, one warp per row: lane cb
// holds columns cb, cb + 32, ... of row g*kR + r of S, so that a warp touches
// 32 consecutive words of shared memory.  Writes o [B][T][H][D] and the state
// before every chunk of kC tokens.  The next chunk's q^, k^, v^ rows and
// gates are copied into the other shared buffer while this one is computed.
template <int D>
struct Stage {
    float q[2][kC][D], k[2][kC][D], v[2][kC][kR], la[2][kC], be[2][kC];
};

// thread tid's share of the copies of chunk c into buffer buf (v: rows g*kR ..; dO likewise if given)
template <int D>
__device__ __forceinline__ void stage_chunk(Stage<D> &st, float (*dO)[kC][kR], const BwdParams &p, size_t bh,
                                            int g, int c, int buf, int tid) {
    const int c0 = c * kC;
    for (int e = tid; e < kC * D / 4; e += kBT) {
        const int tt = e / (D / 4), j = (e % (D / 4)) * 4;
        const size_t src = (bh * p.Tp + c0 + tt) * D + j;
        cp_async16(&st.q[buf][tt][j], p.qh + src);
        cp_async16(&st.k[buf][tt][j], p.kh + src);
    }
    if (tid < kC * kR) {
        const size_t src = (bh * p.Tp + c0 + tid / kR) * D + g * kR + tid % kR;
        cp_async4(&st.v[buf][tid / kR][tid % kR], p.vh + src);
        if (dO) cp_async4(&dO[buf][tid / kR][tid % kR], p.dO + src);
    }
    if (tid < kC) {
        cp_async4(&st.la[buf][tid], p.log_alpha + bh * p.Tp + c0 + tid);
        cp_async4(&st.be[buf][tid], p.beta + bh * p.Tp + c0 + tid);
    }
    cp_async_commit();
}

template <int D>
__global__ void __launch_bounds__(kBT) gdn_bwd_fwd_rows(const BwdParams p) {
    constexpr int CW = D / 32;
    __shared__ __align__(16) Stage<D> st;
    const int g = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const size_t bh = static_cast<size_t>(b) * p.H + h;
    const int tid = threadIdx.x, r = tid >> 5, cb = tid & 31;
    const int i = g * kR + r;
    const int NC = (p.T + kC - 1) / kC;
    float S[CW];
#pragma unroll
    for (int e = 0; e < CW; ++e) S[e] = 0.0f;
    stage_chunk<D>(st, nullptr, p, bh, g, 0, 0, tid);
    for (int c = 0; c < NC; ++c) {
        const int c0 = c * kC, n = min(kC, p.T - c0), buf = c & 1;
        if (c + 1 < NC) {
            stage_chunk<D>(st, nullptr, p, bh, g, c + 1, buf ^ 1, tid);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();  // chunk c's rows are visible
        float *ck = p.ckpt + ((bh * NC + c) * D + i) * D + cb;
#pragma unroll
        for (int e = 0; e < CW; ++e) ck[32 * e] = S[e];
        // unrolled over the chunk (n is uniform): token t's output sum overlaps token t + 1's update
#pragma unroll
        for (int tt = 0; tt < kC; ++tt) {
            if (tt >= n) break;
            const float a = expf(st.la[buf][tt]), be = st.be[buf][tt];
            float u = 0.0f;
#pragma unroll
            for (int e = 0; e < CW; ++e) u = fmaf(S[e], st.k[buf][tt][cb + 32 * e], u);
            u = rowsum(u);
            const float dl = be * (st.v[buf][tt][r] - a * u);
            float ov = 0.0f;
#pragma unroll
            for (int e = 0; e < CW; ++e) {
                S[e] = fmaf(a, S[e], dl * st.k[buf][tt][cb + 32 * e]);
                ov = fmaf(S[e], st.q[buf][tt][cb + 32 * e], ov);
            }
            ov = rowsum(ov);
            if (cb == 0) p.o[((static_cast<size_t>(b) * p.T + c0 + tt) * p.H + h) * D + i] = ov;
        }
        __syncthreads();  // buffer buf is read out before chunk c + 2 is copied into it
    }
}

// four consecutive 16-bit or fp32 values as fp32 (8- or 16-byte aligned)
template <typename InT>
__device__ __forceinline__ void ld4_in(const InT *src, float (&v)[4]);
template <>
__device__ __forceinline__ void ld4_in<float>(const float *src, float (&v)[4]) {
    const float4 x = *reinterpret_cast<const float4 *>(src);
    v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
}
template <>
__device__ __forceinline__ void ld4_in<__nv_bfloat16>(const __nv_bfloat16 *src, float (&v)[4]) {
    const uint2 u = *reinterpret_cast<const uint2 *>(src);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
    v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
}
template <>
__device__ __forceinline__ void ld4_in<__half>(const __half *src, float (&v)[4]) {
    const uint2 u = *reinterpret_cast<const uint2 *>(src);
    const float2 a = __half22float2(*reinterpret_cast<const __half2 *>(&u.x));
    const float2 b = __half22float2(*reinterpret_cast<const __half2 *>(&u.y));
    v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
}

// ------------------------------------------------------------ output step backwards
// One warp per (b, t, h) row.  y = o rn w SiLU(z), rn = 1/sqrt(mean(o^2) + eps):
//   gz = dy w SiLU(z);  do = rn gz - o rn^3 (o . gz) / D;  dz = dy o rn w SiLU'(z);
//   dw += dy o rn SiLU(z)  (per-CTA partial sums, in a fixed order).
template <typename ZT, typename YT, int D>
__global__ void __launch_bounds__(256) gdn_bwd_out(const BwdParams p) {
    constexpr int PER = D / 32;
    __shared__ float sw[8][D];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const long long nrows = static_cast<long long>(p.B) * p.T * p.H;
    float w[PER], dw[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) {
        w[e] = p.norm_w[lane * PER + e];
        dw[e] = 0.0f;
    }
    const ZT *z = static_cast<const ZT *>(p.z);
    const YT *dy = static_cast<const YT *>(p.dy);
    for (long long row = blockIdx.x * 8ll + warp; row < nrows; row += gridDim.x * 8ll) {
        const long long tok = row / p.H;  // b * T + t
        const int hh = static_cast<int>(row % p.H);
        const int bb = static_cast<int>(tok / p.T), t = static_cast<int>(tok % p.T);
        float ov[PER], zv[PER], gv[PER], sz[PER];
        float ss = 0.0f;
#pragma unroll
        for (int e = 0; e < PER; ++e) {
            const int c = lane * PER + e;
            ov[e] = p.o[row * D + c];
            zv[e] = ldf<ZT>(z + tok * p.tok_stride + static_cast<long long>(hh) * D + c);
            gv[e] = ldf<YT>(dy + row * D + c);
            ss = fmaf(ov[e], ov[e], ss);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        const float rn = 1.0f / sqrtf(ss / D + p.norm_eps);
        float og = 0.0f;
#pragma unroll
        for (int e = 0; e < PER; ++e) {
            sz[e] = zv[e] * sigm(zv[e]);
            og = fmaf(ov[e], gv[e] * w[e] * sz[e], og);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) og += __shfl_xor_sync(0xffffffffu, og, off);
        const float k3 = rn * rn * rn * og / D;
        const size_t bhr = static_cast<size_t>(bb) * p.H + hh;
#pragma unroll
        for (int e = 0; e < PER; ++e) {
            const int c = lane * PER + e;
            const float gz = gv[e] * w[e] * sz[e];
            p.dO[(bhr * p.Tp + t) * D + c] = rn * gz - ov[e] * k3;
            p.dz[row * D + c] = gv[e] * ov[e] * rn * w[e] * dsilu(zv[e]);
            dw[e] = fmaf(gv[e] * ov[e] * rn, sz[e], dw[e]);
        }
    }
#pragma unroll
    for (int e = 0; e < PER; ++e) sw[warp][lane * PER + e] = dw[e];
    __syncthreads();
    for (int c = threadIdx.x; c < D; c += 256) {
        float s = 0.0f;
        for (int k = 0; k < 8; ++k) s += sw[k][c];
        p.dnw_part[static_cast<size_t>(blockIdx.x) * D + c] = s;
    }
}

// The output step backwards for the tensor-core backward (d = 128, dO in fp16): one warp per
// (b, t, h) row, lane l on columns 4l .. 4l+3 with 8- and 16-byte loads and stores, two rows per
// warp step (both rows' loads in flight before either is used), SiLU's sigmoid once per element.
template <typename ZT, typename YT>
__global__ void __launch_bounds__(256, 4) gdn_bwd_out_rows(const BwdParams p) {
    constexpr int D = 128;
    __shared__ float sw[8][D];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, c0 = lane * 4;
    const int nrows = p.B * p.T * p.H;  // < 2^31: the plan bounds B * H * Tp
    float w[4], dw[4];
    ld4_in<float>(p.norm_w + c0, w);
#pragma unroll
    for (int e = 0; e < 4; ++e) dw[e] = 0.0f;
    const ZT *z = static_cast<const ZT *>(p.z);
    const YT *dy = static_cast<const YT *>(p.dy);
    const int stride = gridDim.x * 16;
    for (int r0 = blockIdx.x * 16 + warp * 2; r0 < nrows; r0 += stride) {
        float ov[2][4], zv[2][4], gv[2][4];
        int tokv[2], hv[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int row = r0 + i;
            tokv[i] = row / p.H;
            hv[i] = row - tokv[i] * p.H;
            if (row < nrows) {
                ld4_in<float>(p.o + static_cast<size_t>(row) * D + c0, ov[i]);
                ld4_in<ZT>(z + static_cast<size_t>(tokv[i]) * p.tok_stride + hv[i] * D + c0, zv[i]);
                ld4_in<YT>(dy + static_cast<size_t>(row) * D + c0, gv[i]);
            } else {
#pragma unroll
                for (int e = 0; e < 4; ++e) ov[i][e] = zv[i][e] = gv[i][e] = 0.0f;
            }
        }
        float ss[2], og[2], sg[2][4], sz[2][4];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            ss[i] = 0.0f;
            og[i] = 0.0f;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                sg[i][e] = __fdividef(1.0f, 1.0f + __expf(-zv[i][e]));
                sz[i][e] = zv[i][e] * sg[i][e];
                ss[i] = fmaf(ov[i][e], ov[i][e], ss[i]);
                og[i] = fmaf(ov[i][e], gv[i][e] * w[e] * sz[i][e], og[i]);
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                ss[i] += __shfl_xor_sync(0xffffffffu, ss[i], off);
                og[i] += __shfl_xor_sync(0xffffffffu, og[i], off);
            }
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int row = r0 + i;
            if (row >= nrows) break;
            const int bb = tokv[i] / p.T, t = tokv[i] - bb * p.T;
            const float rn = rsqrtf(ss[i] * (1.0f / D) + p.norm_eps);
            const float k3 = rn * rn * rn * og[i] * (1.0f / D);
            float d[4], dzv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                d[e] = rn * gv[i][e] * w[e] * sz[i][e] - ov[i][e] * k3;
                dzv[e] = gv[i][e] * ov[i][e] * rn * w[e] * sg[i][e] * (1.0f + zv[i][e] * (1.0f - sg[i][e]));
                dw[e] = fmaf(gv[i][e] * ov[i][e] * rn, sz[i][e], dw[e]);
            }
            const size_t bhr = static_cast<size_t>(bb) * p.H + hv[i];
            *reinterpret_cast<uint2 *>(p.dO16 + (bhr * p.Tp + t) * D + c0) =
                make_uint2(pack_half2(d[0], d[1]), pack_half2(d[2], d[3]));
            *reinterpret_cast<float4 *>(p.dz + static_cast<size_t>(row) * D + c0) = make_float4(dzv[0], dzv[1], dzv[2], dzv[3]);
        }
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) sw[warp][c0 + e] = dw[e];
    __syncthreads();
    for (int c = threadIdx.x; c < D; c += 256) {
        float s = 0.0f;
        for (int k = 0; k < 8; ++k) s += sw[k][c];
        p.dnw_part[static_cast<size_t>(blockIdx.x) * D + c] = s;
    }
}

// ------------------------------------------------------------ the recurrence backwards
// Same CTA layout as gdn_bwd_fwd_rows.  Per chunk of kC tokens, last chunk
// first: the states before each token (and after the last) are recomputed
// from the checkpoint into S, the gradient D runs backwards through the chunk
// (kept in registers across chunks, each D_t also stored in Dg), and the row
// sums of the chunk are then taken from shared memory.  The next chunk's
// inputs (and, in registers, its checkpoint) are fetched during this one.
template <int D>
struct CoreSmem {
    float S[kC + 1][kR][D];  // slot s: state before token c0 + s
    float Dg[kC][kR][D];     // D_t after do_t q^_t^T is added
    Stage<D> st;
    float dO[2][kC][kR];
    float u[kC][kR], dl[kC][kR], ddl[kC][kR], du[kC][kR];
    float part[kC][kBT];     // per-thread pieces of <D_t, S_{t-1}>
};

template <int D>
__global__ void __launch_bounds__(kBT) gdn_bwd_core(const BwdParams p) {
    constexpr int CW = D / 32;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    CoreSmem<D> &sm = *reinterpret_cast<CoreSmem<D> *>(smem_raw);
    const int g = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const size_t bh = static_cast<size_t>(b) * p.H + h;
    const size_t BH = static_cast<size_t>(p.B) * p.H;
    const int tid = threadIdx.x, r = tid >> 5, cb = tid & 31;
    const int i = g * kR + r;
    const int NC = (p.T + kC - 1) / kC;
    float Dr[CW], ckn[CW];
#pragma unroll
    for (int e = 0; e < CW; ++e) Dr[e] = 0.0f;
    auto load_ck = [&](int c) {
        const float *ck = p.ckpt + ((bh * NC + c) * D + i) * D + cb;
#pragma unroll
        for (int e = 0; e < CW; ++e) ckn[e] = ck[32 * e];
    };
    stage_chunk<D>(sm.st, sm.dO, p, bh, g, NC - 1, (NC - 1) & 1, tid);
    load_ck(NC - 1);
    for (int c = NC - 1; c >= 0; --c) {
        const int c0 = c * kC, n = min(kC, p.T - c0), buf = c & 1;
        float S[CW];
#pragma unroll
        for (int e = 0; e < CW; ++e) S[e] = ckn[e];
        if (c > 0) {
            stage_chunk<D>(sm.st, sm.dO, p, bh, g, c - 1, buf ^ 1, tid);
            load_ck(c - 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();  // chunk c's inputs are visible; the previous chunk's row sums are done
        const Stage<D> &st = sm.st;
        // states of the chunk
#pragma unroll
        for (int tt = 0; tt < kC; ++tt) {
            if (tt >= n) break;
            const float a = expf(st.la[buf][tt]), be = st.be[buf][tt];
            float u = 0.0f;
#pragma unroll
            for (int e = 0; e < CW; ++e) {
                sm.S[tt][r][cb + 32 * e] = S[e];
                u = fmaf(S[e], st.k[buf][tt][cb + 32 * e], u);
            }
            u = rowsum(u);
            const float dl = be * (st.v[buf][tt][r] - a * u);
#pragma unroll
            for (int e = 0; e < CW; ++e) S[e] = fmaf(a, S[e], dl * st.k[buf][tt][cb + 32 * e]);
            if (cb == 0) {
                sm.u[tt][r] = u;
                sm.dl[tt][r] = dl;
            }
        }
#pragma unroll
        for (int e = 0; e < CW; ++e) sm.S[n][r][cb + 32 * e] = S[e];
        // the gradient, backwards through the chunk
#pragma unroll
        for (int t2 = kC - 1; t2 >= 0; --t2) {
            const int tt = t2 - (kC - n);  // tokens n-1 .. 0
            if (tt < 0) break;
            const float a = expf(st.la[buf][tt]), be = st.be[buf][tt];
            const float dov = sm.dO[buf][tt][r];
            float ddl = 0.0f, pr = 0.0f;
#pragma unroll
            for (int e = 0; e < CW; ++e) {
                Dr[e] = fmaf(dov, st.q[buf][tt][cb + 32 * e], Dr[e]);
                sm.Dg[tt][r][cb + 32 * e] = Dr[e];
                ddl = fmaf(Dr[e], st.k[buf][tt][cb + 32 * e], ddl);
                pr = fmaf(Dr[e], sm.S[tt][r][cb + 32 * e], pr);
            }
            ddl = rowsum(ddl);
            sm.part[tt][tid] = pr;
            const float du = -a * be * ddl;
            if (cb == 0) {
                sm.ddl[tt][r] = ddl;
                sm.du[tt][r] = du;
                p.dvh[(bh * p.Tp + c0 + tt) * D + i] = be * ddl;
            }
#pragma unroll
            for (int e = 0; e < CW; ++e) Dr[e] = fmaf(a, Dr[e], du * st.k[buf][tt][cb + 32 * e]);
        }
        __syncthreads();
        // row sums of the chunk (this group's part)
        for (int e = tid; e < n * D; e += kBT) {
            const int tt = e / D, j = e % D;
            float dq = 0.0f, dk = 0.0f;
#pragma unroll
            for (int rr = 0; rr < kR; ++rr) {
                dq = fmaf(sm.S[tt + 1][rr][j], sm.dO[buf][tt][rr], dq);
                dk = fmaf(sm.Dg[tt][rr][j], sm.dl[tt][rr], dk);
                dk = fmaf(sm.S[tt][rr][j], sm.du[tt][rr], dk);
            }
            const size_t dst = ((g * BH + bh) * p.Tp + c0 + tt) * D + j;
            p.dq_part[dst] = dq;
            p.dk_part[dst] = dk;
        }
        const int warp = tid >> 5, lane = tid & 31;
        for (int tt = warp; tt < n; tt += kBT / 32) {
            float s = 0.0f;
#pragma unroll
            for (int q = 0; q < kBT / 32; ++q) s += sm.part[tt][lane + 32 * q];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
            if (lane == 0) {
                const float a = expf(st.la[buf][tt]), be = st.be[buf][tt];
                float ud = 0.0f, db = 0.0f;
                for (int rr = 0; rr < kR; ++rr) {
                    ud = fmaf(sm.u[tt][rr], sm.ddl[tt][rr], ud);
                    db = fmaf(sm.ddl[tt][rr], st.v[buf][tt][rr] - a * sm.u[tt][rr], db);
                }
                const size_t dst = (g * BH + bh) * p.Tp + c0 + tt;
                p.da_part[dst] = s - be * ud;
                p.db_part[dst] = db;
            }
        }
        __syncthreads();  // buffer buf and the chunk arrays are read out before they are refilled
    }
}

// ------------------------------------------------------------ per-token backwards
// One CTA per (64-token tile, h, b), 256 threads = CPR channel groups of 8 x
// runs of tokens.  For q, k, v in turn: dq^ / dk^ = the sum of the groups'
// parts (dv^ is whole); back through the L2 norm (q^ carries 1/sqrt(d_k)) and
// SiLU into da for the tile's tokens and the 3 after it (conv recomputed from
// the inputs); then dx[t] = sum_k w_k da[t+3-k] and the conv-weight sums of the
// tile.  Threads 0..63 also take the gates of the tile's tokens.
template <typename InT, int D>
__global__ void __launch_bounds__(256) gdn_bwd_tokens(const BwdParams p) {
    constexpr int CPR = D / 8, RG = 256 / CPR;
    __shared__ float sda[kTile + 3][D];
    __shared__ float sred[RG][32];  // conv-weight partials of one channel group, reduced over runs
    __shared__ float sg[2][2];
    const int tile = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const size_t bh = static_cast<size_t>(b) * p.H + h;
    const size_t BH = static_cast<size_t>(p.B) * p.H;
    const int t0 = tile * kTile;
    const int tid = threadIdx.x, cg = tid % CPR, rg = tid / CPR, c0 = cg * 8;
    const int G = p.groups;
    const int ntile = p.Tp / kTile;

    for (int which = 0; which < 3; ++which) {
        const InT *x = static_cast<const InT *>(which == 0 ? p.q : (which == 1 ? p.k : p.v));
        const float *w = which == 0 ? p.conv_q : (which == 1 ? p.conv_k : p.conv_v);
        float *dx = which == 0 ? p.dq : (which == 1 ? p.dk : p.dv);
        float wt[8][4];
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
            const float4 t4 = reinterpret_cast<const float4 *>(w)[static_cast<size_t>(h) * D + c0 + cc];
            wt[cc][0] = t4.x; wt[cc][1] = t4.y; wt[cc][2] = t4.z; wt[cc][3] = t4.w;
        }
        auto xat = [&](int t, int cc) -> float {
            return (t >= 0 && t < p.T)
                       ? ldf<InT>(x + (static_cast<size_t>(b) * p.T + t) * p.tok_stride + static_cast<size_t>(h) * D + c0 + cc)
                       : 0.0f;
        };
        __syncthreads();  // the previous tensor's reads of sda are done
        // every thread runs the same number of steps (the row sums below shuffle across lanes)
        for (int m = 0; m < (kTile + 3 + RG - 1) / RG; ++m) {
            const int tt = rg + m * RG;
            const bool inside = tt < kTile + 3;
            const int t = t0 + tt;
            float a[8], s[8], dh[8];
            float ss = 0.0f;
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) {
                float acc = 0.0f;
#pragma unroll
                for (int k = 0; k < 4; ++k) acc = fmaf(wt[cc][k], xat(t - 3 + k, cc), acc);
                a[cc] = acc;
                s[cc] = acc * sigm(acc);
                ss = fmaf(s[cc], s[cc], ss);
                dh[cc] = 0.0f;
            }
            const bool live = inside && t < p.T;
            if (live) {
                if (which < 2) {
                    const float *part = which == 0 ? p.dq_part : p.dk_part;
                    for (int gg = 0; gg < G; ++gg) {
                        const float *src = part + ((gg * BH + bh) * p.Tp + t) * D + c0;
                        const float4 x0 = reinterpret_cast<const float4 *>(src)[0];
                        const float4 x1 = reinterpret_cast<const float4 *>(src)[1];
                        dh[0] += x0.x; dh[1] += x0.y; dh[2] += x0.z; dh[3] += x0.w;
                        dh[4] += x1.x; dh[5] += x1.y; dh[6] += x1.z; dh[7] += x1.w;
                    }
                } else {
                    const float *src = p.dvh + (bh * p.Tp + t) * D + c0;
#pragma unroll
                    for (int cc = 0; cc < 8; ++cc) dh[cc] = src[cc];
                }
            }
            if (which < 2) {
#pragma unroll
                for (int off = CPR / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
                const float nrm = sqrtf(ss + p.l2_eps);
                const float sc = which == 0 ? p.q_scale : 1.0f;
                float proj = 0.0f;
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) proj = fmaf(s[cc] / nrm, dh[cc], proj);
#pragma unroll
                for (int off = CPR / 2; off > 0; off >>= 1) proj += __shfl_xor_sync(0xffffffffu, proj, off);
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) dh[cc] = sc * (dh[cc] - (s[cc] / nrm) * proj) / nrm;
            }
            if (inside) {
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) sda[tt][c0 + cc] = live ? dh[cc] * dsilu(a[cc]) : 0.0f;
            }
        }
        __syncthreads();
        float dw[8][4];
#pragma unroll
        for (int cc = 0; cc < 8; ++cc)
#pragma unroll
            for (int k = 0; k < 4; ++k) dw[cc][k] = 0.0f;
        for (int tt = rg; tt < kTile; tt += RG) {
            const int t = t0 + tt;
            if (t >= p.T) break;
            float o8[8];
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) {
                float acc = 0.0f;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    acc = fmaf(wt[cc][k], sda[tt + 3 - k][c0 + cc], acc);
                    dw[cc][k] = fmaf(sda[tt][c0 + cc], xat(t - 3 + k, cc), dw[cc][k]);
                }
                o8[cc] = acc;
            }
            float *dst = dx + (static_cast<size_t>(b) * p.T + t) * p.H * D + static_cast<size_t>(h) * D + c0;
            reinterpret_cast<float4 *>(dst)[0] = make_float4(o8[0], o8[1], o8[2], o8[3]);
            reinterpret_cast<float4 *>(dst)[1] = make_float4(o8[4], o8[5], o8[6], o8[7]);
        }
        // conv-weight sums over the tile: reduce the RG runs, one channel group at a time
        float *out = p.dconv_part + ((static_cast<size_t>(b) * ntile + tile) * 3 + which) * static_cast<size_t>(p.H) * D * 4;
        for (int q = 0; q < CPR; ++q) {
            __syncthreads();
            if (cg == q) {
#pragma unroll
                for (int cc = 0; cc < 8; ++cc)
#pragma unroll
                    for (int k = 0; k < 4; ++k) sred[rg][cc * 4 + k] = dw[cc][k];
            }
            __syncthreads();
            if (tid < 32) {
                float s = 0.0f;
                for (int rr = 0; rr < RG; ++rr) s += sred[rr][tid];
                out[(static_cast<size_t>(h) * D + q * 8) * 4 + tid] = s;
            }
        }
    }

    // gates: log alpha = -exp(A_log) softplus(g + dt_bias), beta = sigmoid(b)
    float dla_la = 0.0f, dgv = 0.0f;
    if (tid < kTile) {
        const int t = t0 + tid;
        if (t < p.T) {
            float da = 0.0f, db = 0.0f;
            for (int gg = 0; gg < G; ++gg) {
                da += p.da_part[(gg * BH + bh) * p.Tp + t];
                db += p.db_part[(gg * BH + bh) * p.Tp + t];
            }
            const size_t gi = (static_cast<size_t>(b) * p.T + t) * p.H + h;
            const float xg = p.g[gi] + p.dt_bias[h];
            const float eA = expf(p.A_log[h]);
            const float la = -eA * softplus_f(xg);
            const float dla = p.tc ? da : da * expf(la);  // d log alpha (given, or from d alpha)
            dgv = dla * (-eA * sigm(xg));
            dla_la = dla * la;
            const float be = sigm(p.bg[gi]);
            p.dg[gi] = dgv;
            p.db[gi] = db * be * (1.0f - be);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            dla_la += __shfl_xor_sync(0xffffffffu, dla_la, off);
            dgv += __shfl_xor_sync(0xffffffffu, dgv, off);
        }
        if ((tid & 31) == 0) {
            sg[tid >> 5][0] = dla_la;
            sg[tid >> 5][1] = dgv;
        }
    }
    __syncthreads();
    if (tid == 0) {
        const size_t k = (static_cast<size_t>(b) * p.H + h) * ntile + tile;
        p.dA_part[k] = sg[0][0] + sg[1][0];
        p.ddt_part[k] = sg[0][1] + sg[1][1];
    }
}

// ------------------------------------------------------------ per-token backwards, one warp per row
// The tensor-core backward's per-token step (d = 128, whole dq^ / dk^ / dv^ and d log alpha).  One
// CTA per (64-token tile, h, b), 8 warps, lane l on channels 4l .. 4l+3 of a token row.  For q, k, v
// in turn: pass 1 takes the tile's tokens and the 3 after it, one token per warp at a time (the rows
// are independent): the conv of the 4 input rows, SiLU, the L2-norm sums as warp reductions, and
// da = dL/d(conv output) into shared memory; pass 2 takes the tile's tokens again for
// dx[t] = sum_k w_k da[t+3-k] and the conv-weight sums (input rows re-read, from L1), reduced over
// the warps in a fixed order into the tile's partial slot.  Then the gates of the tile's tokens.
template <typename InT>
__global__ void __launch_bounds__(256) gdn_bwd_tokens_rows(const BwdParams p) {
    constexpr int D = 128, NR = kTile + 3;
    __shared__ float4 sda[NR][32];    // da of token t0 + tt, channels 4 lane .. 4 lane + 3
    __shared__ float4 swt[4][32];     // conv taps of channel 4 lane + j
    __shared__ float sg[8][2];
    // per-warp conv-weight sums of channel 4 lane + j, over sda once pass 2 has read it
    float4 (*sdw)[4][32] = reinterpret_cast<float4 (*)[4][32]>(&sda[0][0]);
    static_assert(sizeof(sda) >= 8 * 4 * 32 * sizeof(float4), "the warp sums fit in sda");
    const int tile = blockIdx.x, h = blockIdx.y, b = blockIdx.z / 3, which = blockIdx.z % 3;
    const size_t bh = static_cast<size_t>(b) * p.H + h;
    const int t0 = tile * kTile;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, c0 = lane * 4;
    const int ntile = p.Tp / kTile;
    {
        const InT *x = static_cast<const InT *>(which == 0 ? p.q : (which == 1 ? p.k : p.v));
        const float *wc = which == 0 ? p.conv_q : (which == 1 ? p.conv_k : p.conv_v);
        const float *dh_src = which == 0 ? p.dq_part : (which == 1 ? p.dk_part : p.dvh);
        float *dx = which == 0 ? p.dq : (which == 1 ? p.dk : p.dv);
        const float sc = which == 0 ? p.q_scale : 1.0f;
        auto xrow = [&](int t, float (&v)[4]) {
            if (t >= 0 && t < p.T) {
                ld4_in<InT>(x + (static_cast<size_t>(b) * p.T + t) * p.tok_stride + static_cast<size_t>(h) * D + c0, v);
            } else {
                v[0] = v[1] = v[2] = v[3] = 0.0f;
            }
        };
        if (warp < 4) swt[warp][lane] = reinterpret_cast<const float4 *>(wc)[static_cast<size_t>(h) * D + c0 + warp];
        __syncthreads();
        // conv taps read from shared memory at each use
        auto wt = [&](int j) { return swt[j][lane]; };
        // pass 1: da of tokens t0 .. t0 + 66 (zero past T), in runs of two consecutive tokens taken by the
        // warps in turn: a run's 5 input rows and 2 gradient rows are fetched before any is used, and
        // the two tokens' reductions are independent
        for (int rb = 2 * warp; rb < NR; rb += 16) {
            float xr[5][4], dh[2][4];
#pragma unroll
            for (int k = 0; k < 5; ++k) xrow(t0 + rb - 3 + k, xr[k]);
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int t = t0 + rb + i;
                if (t < p.T && rb + i < NR) {
                    ld4_in<float>(dh_src + (bh * p.Tp + t) * D + c0, dh[i]);
                } else {
                    dh[i][0] = dh[i][1] = dh[i][2] = dh[i][3] = 0.0f;
                }
            }
            // sigma(a) once per element (fast exponential and division); SiLU' = sigma (1 + a (1 - sigma))
            float a[2][4], sg[2][4], sv[2][4], ss[2], pr[2];
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                ss[i] = 0.0f;
                pr[i] = 0.0f;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float4 w4 = wt(j);
                    a[i][j] = w4.x * xr[i][j] + w4.y * xr[i + 1][j] + w4.z * xr[i + 2][j] + w4.w * xr[i + 3][j];
                    sg[i][j] = __fdividef(1.0f, 1.0f + __expf(-a[i][j]));
                    sv[i][j] = a[i][j] * sg[i][j];
                    ss[i] = fmaf(sv[i][j], sv[i][j], ss[i]);
                    pr[i] = fmaf(sv[i][j], dh[i][j], pr[i]);
                }
            }
            if (which < 2) {
                // with u = s / n, n = sqrt(|s|^2 + eps): d s = sc (dh - u (u . dh)) / n
#pragma unroll
                for (int off = 16; off > 0; off >>= 1)
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        ss[i] += __shfl_xor_sync(0xffffffffu, ss[i], off);
                        pr[i] += __shfl_xor_sync(0xffffffffu, pr[i], off);
                    }
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const float inv = rsqrtf(ss[i] + p.l2_eps);
                    const float k2 = inv * inv * pr[i];
#pragma unroll
                    for (int j = 0; j < 4; ++j) dh[i][j] = sc * inv * (dh[i][j] - sv[i][j] * k2);
                }
            }
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int t = t0 + rb + i;
                if (rb + i < NR) {
                    float da[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        da[j] = t < p.T ? dh[i][j] * sg[i][j] * (1.0f + a[i][j] * (1.0f - sg[i][j])) : 0.0f;
                    sda[rb + i][lane] = make_float4(da[0], da[1], da[2], da[3]);
                }
            }
        }
        __syncthreads();
        // pass 2: dx[t] = sum_k w_k da[t + 3 - k] and the conv-weight sums (tap k multiplies x[t - 3 + k])
        float dw[4][4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int k = 0; k < 4; ++k) dw[j][k] = 0.0f;
        for (int tt = warp; tt < kTile; tt += 8) {
            const int t = t0 + tt;
            if (t >= p.T) break;
            float dr[4][4], xr[4][4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float4 v = sda[tt + k][lane];
                dr[k][0] = v.x; dr[k][1] = v.y; dr[k][2] = v.z; dr[k][3] = v.w;
                xrow(t - 3 + k, xr[k]);
            }
            float o[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float4 w4 = wt(j);
                o[j] = w4.x * dr[3][j] + w4.y * dr[2][j] + w4.z * dr[1][j] + w4.w * dr[0][j];
#pragma unroll
                for (int k = 0; k < 4; ++k) dw[j][k] = fmaf(dr[0][j], xr[k][j], dw[j][k]);
            }
            *reinterpret_cast<float4 *>(dx + (static_cast<size_t>(b) * p.T + t) * p.H * D + static_cast<size_t>(h) * D + c0) =
                make_float4(o[0], o[1], o[2], o[3]);
        }
        __syncthreads();  // every read of sda is done
#pragma unroll
        for (int j = 0; j < 4; ++j) sdw[warp][j][lane] = make_float4(dw[j][0], dw[j][1], dw[j][2], dw[j][3]);
        __syncthreads();
        if (warp < 4) {  // warp j: channel 4 lane + j, the 8 warps' sums in order
            float4 acc = sdw[0][warp][lane];
#pragma unroll
            for (int k = 1; k < 8; ++k) {
                const float4 v = sdw[k][warp][lane];
                acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
            }
            float *out = p.dconv_part + ((static_cast<size_t>(b) * ntile + tile) * 3 + which) * static_cast<size_t>(p.H) * D * 4 +
                         (static_cast<size_t>(h) * D + c0 + warp) * 4;
            *reinterpret_cast<float4 *>(out) = acc;
        }
    }

    // gates (the q CTA of the tile): log alpha = -exp(A_log) softplus(g + dt_bias), beta = sigmoid(b);
    // d log alpha is given
    if (which != 0) return;
    float dla_la = 0.0f, dgv = 0.0f;
    if (threadIdx.x < kTile) {
        const int t = t0 + threadIdx.x;
        if (t < p.T) {
            const float eA = expf(p.A_log[h]);
            const float dla = p.da_part[bh * p.Tp + t];
            const float db = p.db_part[bh * p.Tp + t];
            const size_t gi = (static_cast<size_t>(b) * p.T + t) * p.H + h;
            const float xg = p.g[gi] + p.dt_bias[h];
            const float la = -eA * softplus_f(xg);
            const float dg = dla * (-eA * sigm(xg));
            dgv = dg;
            dla_la = dla * la;
            const float be = sigm(p.bg[gi]);
            p.dg[gi] = dg;
            p.db[gi] = db * be * (1.0f - be);
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        dla_la += __shfl_xor_sync(0xffffffffu, dla_la, off);
        dgv += __shfl_xor_sync(0xffffffffu, dgv, off);
    }
    if (lane == 0) {
        sg[warp][0] = dla_la;
        sg[warp][1] = dgv;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const size_t k = bh * ntile + tile;
        p.dA_part[k] = sg[0][0] + sg[1][0];
        p.ddt_part[k] = sg[0][1] + sg[1][1];
    }
}

// ------------------------------------------------------------ parameter sums
// 32 parameter gradient elements per CTA, 8 warps: warp g sums partials g, g + 8, ... of lane l's
// element, then the 8 warp sums are added in order (a fixed order throughout).
__global__ void __launch_bounds__(256) gdn_bwd_params_split(const BwdParams p, int D, int nout_part) {
    __shared__ float red[8][32];
    const int HD4 = p.H * D * 4;
    const int ntile = p.Tp / kTile;
    const int total = 3 * HD4 + 2 * p.H + D;
    const int lane = threadIdx.x & 31, g = threadIdx.x >> 5;
    const int e = blockIdx.x * 32 + lane;
    float sum = 0.0f;
    if (e < 3 * HD4) {
        const int which = e / HD4, k = e % HD4;
        for (int bt = g; bt < p.B * ntile; bt += 8) sum += p.dconv_part[(static_cast<size_t>(bt) * 3 + which) * HD4 + k];
    } else if (e < 3 * HD4 + 2 * p.H) {
        const int k = e - 3 * HD4, h = k % p.H;
        const float *part = k < p.H ? p.dA_part : p.ddt_part;
        for (int i = g; i < p.B * ntile; i += 8) {
            const int b = i / ntile, t = i % ntile;
            sum += part[(static_cast<size_t>(b) * p.H + h) * ntile + t];
        }
    } else if (e < total) {
        const int c = e - 3 * HD4 - 2 * p.H;
        for (int q = g; q < nout_part; q += 8) sum += p.dnw_part[static_cast<size_t>(q) * D + c];
    }
    red[g][lane] = sum;
    __syncthreads();
    if (g == 0 && e < total) {
        float s = 0.0f;
#pragma unroll
        for (int k = 0; k < 8; ++k) s += red[k][lane];
        if (e < 3 * HD4) {
            const int which = e / HD4, k = e % HD4;
            (which == 0 ? p.dconv_q : (which == 1 ? p.dconv_k : p.dconv_v))[k] = s;
        } else if (e < 3 * HD4 + 2 * p.H) {
            const int k = e - 3 * HD4;
            (k < p.H ? p.dA_log : p.ddt_bias)[k % p.H] = s;
        } else {
            p.dnorm_w[e - 3 * HD4 - 2 * p.H] = s;
        }
    }
}

template <typename ZT, typename YT>
cudaError_t launch_out_bwd(const BwdParams &p, int blocks, cudaStream_t s) {
    if (p.dO16) gdn_bwd_out_rows<ZT, YT><<<blocks, 256, 0, s>>>(p);
    else if (p.d == 128) gdn_bwd_out<ZT, YT, 128><<<blocks, 256, 0, s>>>(p);
    else gdn_bwd_out<ZT, YT, 64><<<blocks, 256, 0, s>>>(p);
    return cudaGetLastError();
}
template <typename ZT>
cudaError_t launch_out_bwd_z(const BwdParams &p, InType yt, int blocks, cudaStream_t s) {
    if (yt == InType::BF16) return launch_out_bwd<ZT, __nv_bfloat16>(p, blocks, s);
    if (yt == InType::F16) return launch_out_bwd<ZT, __half>(p, blocks, s);
    return launch_out_bwd<ZT, float>(p, blocks, s);
}

template <int D>
cudaError_t launch_core_bwd(const BwdParams &p, cudaStream_t s) {
    static SmemOnce once;
    const int bytes = static_cast<int>(sizeof(CoreSmem<D>));
    cudaError_t e = raise_smem_once(once, gdn_bwd_core<D>, bytes);
    if (e != cudaSuccess) return e;
    gdn_bwd_core<D><<<dim3(D / kR, p.H, p.B), kBT, bytes, s>>>(p);
    return cudaGetLastError();
}

template <typename InT>
cudaError_t launch_tokens_bwd(const BwdParams &p, cudaStream_t s) {
    const dim3 grid(p.Tp / kTile, p.H, p.B);
    if (p.d == 128) gdn_bwd_tokens<InT, 128><<<grid, 256, 0, s>>>(p);
    else gdn_bwd_tokens<InT, 64><<<grid, 256, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_out(const BwdParams &p, InType in, InType out, cudaStream_t s) {
    const int nb = bwd_out_blocks(static_cast<long long>(p.B) * p.T * p.H);
    if (in == InType::BF16) return launch_out_bwd_z<__nv_bfloat16>(p, out, nb, s);
    if (in == InType::F16) return launch_out_bwd_z<__half>(p, out, nb, s);
    return launch_out_bwd_z<float>(p, out, nb, s);
}

cudaError_t launch_bwd_tokens(const BwdParams &p, InType in, cudaStream_t s) {
    if (p.tc && p.d == 128) {  // whole per-token gradients: one warp per row
        const dim3 grid(p.Tp / kTile, p.H, p.B * 3);  // one CTA per (tile, head, sequence, tensor)
        if (in == InType::BF16) gdn_bwd_tokens_rows<__nv_bfloat16><<<grid, 256, 0, s>>>(p);
        else if (in == InType::F16) gdn_bwd_tokens_rows<__half><<<grid, 256, 0, s>>>(p);
        else gdn_bwd_tokens_rows<float><<<grid, 256, 0, s>>>(p);
        return cudaGetLastError();
    }
    if (in == InType::BF16) return launch_tokens_bwd<__nv_bfloat16>(p, s);
    if (in == InType::F16) return launch_tokens_bwd<__half>(p, s);
    return launch_tokens_bwd<float>(p, s);
}

cudaError_t launch_bwd_params(const BwdParams &p, cudaStream_t s) {
    const int total = 3 * p.H * p.d * 4 + 2 * p.H + p.d;
    gdn_bwd_params_split<<<(total + 31) / 32, 256, 0, s>>>(p, p.d, bwd_out_blocks(static_cast<long long>(p.B) * p.T * p.H));
    return cudaGetLastError();
}

int bwd_out_blocks(long long rows) {
    long long blocks = (rows + 7) / 8;
    return static_cast<int>(blocks < 4096 ? blocks : 4096);
}

cudaError_t launch_backward(const BwdParams &p, InType in, InType out, cudaStream_t s, int *launches,
                            void *const *events) {
    cudaError_t e;
    int n = 0;
    // events[i] (optional) is recorded before the i-th launch, events[5] after the last
    auto mark = [&](int i) -> cudaError_t {
        return events ? cudaEventRecord(reinterpret_cast<cudaEvent_t>(events[i]), s) : cudaSuccess;
    };
    if ((e = mark(0)) != cudaSuccess) return e;
    const dim3 grid_rows(p.d / kR, p.H, p.B);
    if (p.d == 128) gdn_bwd_fwd_rows<128><<<grid_rows, kBT, 0, s>>>(p);
    else gdn_bwd_fwd_rows<64><<<grid_rows, kBT, 0, s>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    ++n;
    if ((e = mark(1)) != cudaSuccess) return e;
    const int nb = bwd_out_blocks(static_cast<long long>(p.B) * p.T * p.H);
    if (in == InType::BF16) e = launch_out_bwd_z<__nv_bfloat16>(p, out, nb, s);
    else if (in == InType::F16) e = launch_out_bwd_z<__half>(p, out, nb, s);
    else e = launch_out_bwd_z<float>(p, out, nb, s);
    if (e != cudaSuccess) return e;
    ++n;
    if ((e = mark(2)) != cudaSuccess) return e;
    e = p.d == 128 ? launch_core_bwd<128>(p, s) : launch_core_bwd<64>(p, s);
    if (e != cudaSuccess) return e;
    ++n;
    if ((e = mark(3)) != cudaSuccess) return e;
    if (in == InType::BF16) e = launch_tokens_bwd<__nv_bfloat16>(p, s);
    else if (in == InType::F16) e = launch_tokens_bwd<__half>(p, s);
    else e = launch_tokens_bwd<float>(p, s);
    if (e != cudaSuccess) return e;
    ++n;
    if ((e = mark(4)) != cudaSuccess) return e;
    if ((e = launch_bwd_params(p, s)) != cudaSuccess) return e;
    ++n;
    if ((e = mark(5)) != cudaSuccess) return e;
    if (launches) *launches = n;
    return cudaSuccess;
}

}  // namespace gdn

GDN_TRACE_EXPORT(backward)
