// gdn_proj.cu -- the projections around the GDN core on tcgen05: the input
// projection x W_in^T of the hidden states into q, k, v, z, g, b, with the
// short convolution, SiLU and L2 norm of q, k, v done in the GEMM epilogue,
// and the output projection y W_out^T.
//
// Both are one persistent GEMM kernel, C[M][N] = A[M][K] B[N][K]^T with bf16
// (or fp16) operands, both K-major (the row-major activations and the
// [out][in] weight layout of a linear layer), and fp32 accumulation in tensor
// memory:
//   warp 0       TMA producer: 128 x 64 A and 256 x 64 B boxes (128-byte
//                swizzle) into a 4-stage ring of shared-memory slots;
//   warp 1       owns the tensor memory and issues the MMAs (M = 128, N = 256,
//                K = 16 per instruction) into one of two 256-column fp32
//                accumulators, so that a tile's epilogue overlaps the next
//                tile's products;
//   warps 2-17   epilogue: warp w reads TMEM lane quarter w % 4 (rows) of
//                the 64-column quarter (w - 2) / 4 of the tile (half a head).
// Tiles are handed out round-robin, N fastest, so that the CTAs working at one
// time share A rows and the whole weight through L2.
//
// Input-projection epilogue.  N is split into q | k | v | z (H*128 columns
// each, two heads per 256-column tile) and a last tile holding g and b (2H
// columns).  conv4 at token t needs the projections of tokens t-3..t, so an
// M tile covers 128 consecutive rows but advances by 125: its first 3 rows are
// the previous tokens (history only), rows 3..127 are its outputs.  Inside a
// warp the history comes by shuffles; the first 3 lanes of a quarter get the
// last 3 rows of the quarter above through shared memory.  The taps of the
// tile's channels are staged in shared memory once per tile, and the two warps
// holding the halves of a head's row add their sums of squares there.  Taps reaching
// before the start of a batch item read zero, as in the definition.  q and k
// are then L2-normalised over their head (q also scaled by 1/sqrt(d)), and
// q^, k^, v^ are written as fp16 in the tensor path's [B][H][Tp][128]
// operand layout; z goes out as fp16 [B][T][H*128], g and b as fp32 [B][T][H].
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

namespace pj {
constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr uint32_t A_BYTES = BM * BK * 2;              // 16 KB
constexpr uint32_t B_BYTES = BN * BK * 2;              // 32 KB
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
// conv history rows, per (chunk parity, sub, quarter): the last 3 rows of the quarter, 32 values
// each, rows 36 floats apart (16-byte aligned)
constexpr int HALO_SLOT = 112;
constexpr uint32_t OFF_HALO = STAGES * STAGE_BYTES;
constexpr uint32_t HALO_BYTES = 2 * 4 * 4 * HALO_SLOT * 4;
constexpr uint32_t OFF_TAPS = OFF_HALO + HALO_BYTES;   // conv taps of the tile, per sub [4 taps][64 channels]
constexpr uint32_t TAPS_BYTES = 4 * 4 * 64 * 4;
constexpr uint32_t OFF_SS = OFF_TAPS + TAPS_BYTES;     // q/k sums of squares, [tile parity][2 heads][4 quarters][2 parts][32]
constexpr uint32_t SS_BYTES = 2 * 2 * 4 * 2 * 32 * 4;
constexpr uint32_t OFF_BAR = OFF_SS + SS_BYTES;
enum { FULL = 0, EMPTY = STAGES, ACC_FULL = 2 * STAGES, ACC_EMPTY = ACC_FULL + 2, NBAR = ACC_EMPTY + 2 };
constexpr uint32_t SMEM_BYTES = OFF_BAR + NBAR * 8 + 16 + 1024;
constexpr int kEpiWarps = 16;
constexpr int kThreads = 32 * (2 + kEpiWarps);
constexpr int kHist = 3;  // conv history rows at the top of an input-projection M tile
}  // namespace pj

__device__ __forceinline__ void store32_f16(__half *dst, const float (&v)[32], float scale) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint4 u;
        u.x = pack_half2(v[8 * i] * scale, v[8 * i + 1] * scale);
        u.y = pack_half2(v[8 * i + 2] * scale, v[8 * i + 3] * scale);
        u.z = pack_half2(v[8 * i + 4] * scale, v[8 * i + 5] * scale);
        u.w = pack_half2(v[8 * i + 6] * scale, v[8 * i + 7] * scale);
        reinterpret_cast<uint4 *>(dst)[i] = u;
    }
}

__device__ __forceinline__ void store32_bf16(__nv_bfloat16 *dst, const float (&v)[32]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            __nv_bfloat162 b2 = __floats2bfloat162_rn(v[8 * i + 2 * j], v[8 * i + 2 * j + 1]);
            w[j] = *reinterpret_cast<uint32_t *>(&b2);
        }
        reinterpret_cast<uint4 *>(dst)[i] = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

struct EpiSmem {
    float *halo, *taps, *ss;
};

// The input projection's epilogue for one 128-row x 64-column quarter of a tile (this warp's
// lane quarter q; TMEM address tacc = this thread's lane, the quarter's first column).  Row
// r = 32 q + lane is token row m = m0 - 3 + r; sub = 64-column quarter of the 256-column tile
// (head = sub / 2 of the tile's two heads, part = sub % 2 of its 128 columns).
__device__ __forceinline__ void epilogue_in(const ProjParams &p, uint32_t tacc, int mi, int ni, int sub, int q,
                                            int lane, int c_base, int tpar, const EpiSmem &es) {
    using namespace pj;
    const int half = sub >> 1, part = sub & 1;
    const int r = q * 32 + lane;
    const int m = mi * p.m_step - kHist + r;
    const bool out_row = r >= kHist && m < p.M;
    const int bb = m >= 0 ? m / p.T : 0;
    const int tt = m - bb * p.T;  // token within its batch item (valid for m >= 0)
    const int per_tensor = p.H / 2;
    if (ni >= 4 * per_tensor) {
        // g | b tile: columns 0 .. H-1 are g, H .. 2H-1 are b
        const size_t gi = static_cast<size_t>(m) * p.H;
        const bool ok = out_row && debug_in_bounds(p.debug, gi, p.H, static_cast<size_t>(p.M) * p.H, p.status);
        for (int cc = 0; cc < 2 && sub * 64 + 32 * cc < 2 * p.H; ++cc) {
            float x[32];
            tmem_ld32(tacc + 32 * cc, x);
            if (ok) {
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int col = sub * 64 + 32 * cc + e;
                    if (col < p.H) p.g[gi + col] = x[e];
                    else if (col < 2 * p.H) p.b[gi + col - p.H] = x[e];
                }
            }
        }
        return;
    }
    const int tensor = ni / per_tensor;               // 0 q, 1 k, 2 v, 3 z
    const int head = 2 * (ni - tensor * per_tensor) + half;
    const int col0 = part * 64;                       // first column of this quarter within the head
    if (tensor == 3) {                                // z: no conv, fp16 out
        const size_t o = static_cast<size_t>(m) * p.H * kD + static_cast<size_t>(head) * kD + col0;
        const bool ok = out_row && debug_in_bounds(p.debug, o, 64, static_cast<size_t>(p.M) * p.H * kD, p.status);
#pragma unroll 1
        for (int cc = 0; cc < 2; ++cc) {
            float x[32];
            tmem_ld32(tacc + 32 * cc, x);
            if (ok) store32_f16(p.z + o + 32 * cc, x, 1.0f);
        }
        return;
    }
    const float *conv = tensor == 0 ? p.conv_q : (tensor == 1 ? p.conv_k : p.conv_v);
    __half *outp = tensor == 0 ? p.qh : (tensor == 1 ? p.kh : p.vh);
    const size_t orow = (static_cast<size_t>(bb) * p.H + head) * p.Tp + tt;
    const bool ok = out_row && debug_in_bounds(p.debug, orow * kD + col0, 64,
                                               static_cast<size_t>(p.B) * p.H * p.Tp * kD, p.status);
    __half *dst = outp + orow * kD + col0;
    // the taps of this quarter's 64 channels, [tap][channel]; published by the first history barrier
    float *taps = es.taps + sub * 256;
    {
        const int i = q * 32 + lane;  // 0 .. 127 over the sub's four warps
        const float *src = conv + static_cast<size_t>(head * kD + col0) * 4;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int idx = i + 128 * k;  // channel idx / 4, tap idx % 4
            taps[(idx & 3) * 64 + (idx >> 2)] = __ldg(src + idx);
        }
    }
    // taps that reach before the batch item's first token read zero
    const float m1 = tt >= 1 ? 1.0f : 0.0f, m2 = tt >= 2 ? 1.0f : 0.0f, m3 = tt >= 3 ? 1.0f : 0.0f;
    float ss = 0.0f;
#pragma unroll 1
    for (int cc = 0; cc < 2; ++cc) {
        float x[32];
        tmem_ld32(tacc + 32 * cc, x);
        // publish this quarter's last 3 rows for the quarter below; slots alternate by chunk parity
        const int par = (c_base + cc) & 1;
        float *mine = es.halo + ((par * 4 + sub) * 4 + q) * HALO_SLOT;
        const float *prev = es.halo + ((par * 4 + sub) * 4 + ((q + 3) & 3)) * HALO_SLOT;
        if (lane >= 29) {
#pragma unroll
            for (int e4 = 0; e4 < 8; ++e4)
                *reinterpret_cast<float4 *>(mine + (lane - 29) * 36 + 4 * e4) =
                    make_float4(x[4 * e4], x[4 * e4 + 1], x[4 * e4 + 2], x[4 * e4 + 3]);
        }
        named_sync(2 + sub, 128);
        // lane l < j takes row r - j from slot row 3 + l - j of the quarter above (other lanes
        // read a clamped row and discard it)
        const float *h1 = prev + min(2 + lane, 2) * 36, *h2 = prev + min(1 + lane, 2) * 36, *h3 = prev + min(lane, 2) * 36;
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
            const float4 w0 = *reinterpret_cast<const float4 *>(taps + 0 * 64 + 32 * cc + 4 * e4);
            const float4 w1 = *reinterpret_cast<const float4 *>(taps + 1 * 64 + 32 * cc + 4 * e4);
            const float4 w2 = *reinterpret_cast<const float4 *>(taps + 2 * 64 + 32 * cc + 4 * e4);
            const float4 w3 = *reinterpret_cast<const float4 *>(taps + 3 * 64 + 32 * cc + 4 * e4);
            const float4 p1 = *reinterpret_cast<const float4 *>(h1 + 4 * e4);
            const float4 p2 = *reinterpret_cast<const float4 *>(h2 + 4 * e4);
            const float4 p3 = *reinterpret_cast<const float4 *>(h3 + 4 * e4);
            const float w0a[4] = {w0.x, w0.y, w0.z, w0.w}, w1a[4] = {w1.x, w1.y, w1.z, w1.w};
            const float w2a[4] = {w2.x, w2.y, w2.z, w2.w}, w3a[4] = {w3.x, w3.y, w3.z, w3.w};
            const float p1a[4] = {p1.x, p1.y, p1.z, p1.w}, p2a[4] = {p2.x, p2.y, p2.z, p2.w};
            const float p3a[4] = {p3.x, p3.y, p3.z, p3.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int e = 4 * e4 + i;
                const float s1 = __shfl_up_sync(0xffffffffu, x[e], 1);
                const float s2 = __shfl_up_sync(0xffffffffu, x[e], 2);
                const float s3 = __shfl_up_sync(0xffffffffu, x[e], 3);
                const float x1 = (lane < 1 ? p1a[i] : s1) * m1;
                const float x2 = (lane < 2 ? p2a[i] : s2) * m2;
                const float x3 = (lane < 3 ? p3a[i] : s3) * m3;
                float u = w3a[i] * x[e];  // tap 3: the current token
                u = fmaf(w2a[i], x1, u);
                u = fmaf(w1a[i], x2, u);
                u = fmaf(w0a[i], x3, u);
                u = silu_f(u);
                ss = fmaf(u, u, ss);
                x[e] = u;
            }
        }
        if (tensor == 2) {
            if (ok) store32_f16(dst + 32 * cc, x, 1.0f);
        } else {
            tmem_st32(tacc + 32 * cc, x);  // the activated value waits in TMEM for the head's norm
        }
    }
    if (tensor == 2) return;
    // the head's sum of squares: this quarter's 64 columns plus the partner warp's other 64
    float *ssl = es.ss + ((tpar * 2 + half) * 4 + q) * 64;
    ssl[part * 32 + lane] = ss;
    named_sync(6 + half, 256);
    ss += ssl[(part ^ 1) * 32 + lane];
    tmem_st_wait();
    const float sc = rsqrtf(ss + p.l2_eps) * (tensor == 0 ? p.q_scale : 1.0f);
#pragma unroll 1
    for (int cc = 0; cc < 2; ++cc) {
        float x[32];
        tmem_ld32(tacc + 32 * cc, x);
        if (ok) store32_f16(dst + 32 * cc, x, sc);
    }
}

// The output projection's epilogue: row m = m0 + r, columns n0 + 64 sub + 32 cc + e.
__device__ __forceinline__ void epilogue_out(const ProjParams &p, uint32_t tacc, int mi, int ni, int sub, int q,
                                             int lane) {
    const int m = mi * p.m_step + q * 32 + lane;
    const int n0 = ni * pj::BN + sub * 64;
#pragma unroll 1
    for (int cc = 0; cc < 2; ++cc) {
        float x[32];
        tmem_ld32(tacc + 32 * cc, x);
        const int n = n0 + 32 * cc;
        if (m >= p.M || n >= p.N) continue;
        const size_t o = static_cast<size_t>(m) * p.N + n;
        if (!debug_in_bounds(p.debug, o, 32, static_cast<size_t>(p.M) * p.N, p.status)) continue;
        if (p.out_kind == 1) {
            float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(p.out) + o);
#pragma unroll
            for (int i = 0; i < 8; ++i) dst[i] = make_float4(x[4 * i], x[4 * i + 1], x[4 * i + 2], x[4 * i + 3]);
        } else {
            store32_bf16(static_cast<__nv_bfloat16 *>(p.out) + o, x);
        }
    }
}

template <int kMode>  // 0: input projection (conv / SiLU / L2 epilogue), 1: output projection
__global__ void __launch_bounds__(pj::kThreads, 1)
    gdn_proj_kernel(const ProjParams p, const __grid_constant__ CUtensorMap tmA,
                    const __grid_constant__ CUtensorMap tmB) {
    using namespace pj;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + NBAR);
    AbortState *ab = reinterpret_cast<AbortState *>(tmem_slot + 1);
    const EpiSmem es = {reinterpret_cast<float *>(sm + OFF_HALO), reinterpret_cast<float *>(sm + OFF_TAPS),
                        reinterpret_cast<float *>(sm + OFF_SS)};
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ntiles = p.m_tiles * p.n_tiles;
    const int nkb = p.K / BK;
    const uint64_t lim = p.wait_limit_ns;

    if (tid == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&bars[FULL + i], 1);
            mbar_init(&bars[EMPTY + i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars[ACC_FULL + i], 1);
            mbar_init(&bars[ACC_EMPTY + i], kEpiWarps);
        }
        ab->flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    pdl_launch_dependents();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_wait();  // the previous kernel's output (the output projection's A) is complete

    if (warp == 0) {
        if (lane == 0) {
            // phases started on each FULL slot, for the drain at the end (every earlier phase of a
            // slot has been consumed before its next load starts)
            int started[STAGES] = {};
            bool ok = true;
            int it = 0;
            for (int t = blockIdx.x; ok && t < ntiles; t += gridDim.x) {
                const int mi = t / p.n_tiles, ni = t - mi * p.n_tiles;
                const int arow = mi * p.m_step - (kMode == 0 ? kHist : 0);  // negative rows read as zero
                const int brow = ni * BN;
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int s = it % STAGES;
                    ok = mbar_wait(&bars[EMPTY + s], ((it / STAGES) & 1) ^ 1, ab, p.status, lim);
                    if (!ok) break;
                    mbar_arrive_expect_tx(&bars[FULL + s], STAGE_BYTES);
                    tma_load_2d(sm + s * STAGE_BYTES, &tmA, &bars[FULL + s], kb * BK, arow);
                    tma_load_2d(sm + s * STAGE_BYTES + A_BYTES, &tmB, &bars[FULL + s], kb * BK, brow);
                    ++started[s];
                }
            }
#pragma unroll 1
            for (int s = 0; s < STAGES; ++s)
                if (started[s] > 0) mbar_wait_drain(&bars[FULL + s], (started[s] - 1) & 1, lim);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = p.f16 ? idesc_f16_f32(BM, BN, false, false) : idesc_bf16_f32(BM, BN);
            int committed[STAGES + 2] = {};  // commits on EMPTY slots, then on the two ACC_FULL barriers
            bool ok = true;
            int it = 0, local = 0;
            for (int t = blockIdx.x; ok && t < ntiles; t += gridDim.x, ++local) {
                const int buf = local & 1;
                ok = mbar_wait(&bars[ACC_EMPTY + buf], ((local >> 1) & 1) ^ 1, ab, p.status, lim);
                if (!ok) break;
                tc_fence_after();
                const uint32_t dacc = tmem + buf * BN;
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int s = it % STAGES;
                    ok = mbar_wait(&bars[FULL + s], (it / STAGES) & 1, ab, p.status, lim);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t a0 = sbase + s * STAGE_BYTES, b0 = a0 + A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        umma_f16(dacc, sdesc_sw128(a0 + kk * 32, 16, 1024), sdesc_sw128(b0 + kk * 32, 16, 1024),
                                 idesc, (kb | kk) != 0);
                    umma_commit(&bars[EMPTY + s]);  // the slot is free once these products have read it
                    ++committed[s];
                }
                if (!ok) break;
                umma_commit(&bars[ACC_FULL + buf]);
                ++committed[STAGES + buf];
            }
#pragma unroll 1
            for (int s = 0; s < STAGES; ++s)
                if (committed[s] > 0) mbar_wait_drain(&bars[EMPTY + s], (committed[s] - 1) & 1, lim);
#pragma unroll 1
            for (int b2 = 0; b2 < 2; ++b2)
                if (committed[STAGES + b2] > 0)
                    mbar_wait_drain(&bars[ACC_FULL + b2], (committed[STAGES + b2] - 1) & 1, lim);
        }
    } else {
        const int q = warp & 3, sub = (warp - 2) >> 2;
        const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
        int local = 0, chunks = 0;
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++local) {
            const int buf = local & 1;
            const bool w = mbar_wait(&bars[ACC_FULL + buf], (local >> 1) & 1, ab, p.status, lim);
            // all epilogue warps go on, or stop, together: the head-level barrier below joins two subs
            if (!group_all(1, 32 * kEpiWarps, w)) break;
            tc_fence_after();
            const int mi = t / p.n_tiles, ni = t - mi * p.n_tiles;
            const uint32_t tacc = tmem + lane_base + buf * BN + sub * 64;
            if (kMode == 0) {
                epilogue_in(p, tacc, mi, ni, sub, q, lane, chunks, local & 1, es);
                chunks += 2;
            } else {
                epilogue_out(p, tacc, mi, ni, sub, q, lane);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[ACC_EMPTY + buf]);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

// bf16 -> fp16, n elements (n a multiple of 8, both 16-byte aligned): a weight copy in the
// operand type of the output projection.
__global__ void __launch_bounds__(256) gdn_bf16_to_f16_kernel(const uint4 *src, uint4 *dst, size_t n8) {
    for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n8;
         i += static_cast<size_t>(gridDim.x) * blockDim.x) {
        const uint4 u = src[i];
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[j]));
            o[j] = pack_half2(f.x, f.y);
        }
        dst[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

}  // namespace

cudaError_t launch_bf16_to_f16(const void *src, void *dst, size_t n, cudaStream_t s) {
    const size_t n8 = n / 8;
    if (n8 == 0) return cudaSuccess;
    const size_t blocks = (n8 + 255) / 256;
    gdn_bf16_to_f16_kernel<<<static_cast<unsigned>(blocks < 1184 ? blocks : 1184), 256, 0, s>>>(
        static_cast<const uint4 *>(src), static_cast<uint4 *>(dst), n8);
    return cudaGetLastError();
}

cudaError_t launch_proj(const ProjParams &p, int mode, const CUtensorMap &tmA, const CUtensorMap &tmB,
                        cudaStream_t s, bool pdl) {
    static SmemOnce once_in, once_out;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return cudaErrorInvalidDevice;
    const long long ntiles = static_cast<long long>(p.m_tiles) * p.n_tiles;
    if (ntiles < 1) return cudaSuccess;
    const dim3 grid(static_cast<unsigned>(ntiles < sms ? ntiles : sms));
    if (mode == 0) {
        cudaError_t e = raise_smem_once(once_in, gdn_proj_kernel<0>, static_cast<int>(pj::SMEM_BYTES));
        if (e != cudaSuccess) return e;
        return launch_k(gdn_proj_kernel<0>, grid, dim3(pj::kThreads), pj::SMEM_BYTES, s, pdl, p, tmA, tmB);
    }
    cudaError_t e = raise_smem_once(once_out, gdn_proj_kernel<1>, static_cast<int>(pj::SMEM_BYTES));
    if (e != cudaSuccess) return e;
    return launch_k(gdn_proj_kernel<1>, grid, dim3(pj::kThreads), pj::SMEM_BYTES, s, pdl, p, tmA, tmB);
}

int proj_m_step(int mode) { return mode == 0 ? pj::BM - pj::kHist : pj::BM; }
int proj_n_tile() { return pj::BN; }

}  // namespace gdn
