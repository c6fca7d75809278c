// gdn_bwd_tc.cu -- the gradient of the gated delta rule (reference [57] on the
// VMonarch page, with the LinMorph page's decay and update gates) in the block
// (UT / WY) form, on 5th-generation tensor cores, for 16-bit inputs and
// d_k = d_v = 128.
//
// Per 128-token block, with the forward's G (in-block cumulative log decay),
// E = e^G, beta, Q (q^ with 1/sqrt(d_k)), K, V, T = (I + L)^-1,
// W = T diag(beta E) K, U = T diag(beta) V, P = Aqk, Qt = diag(E) Q,
// Kt = diag(e^(G_last - G)) K, the state S0 at the block start and dS = dL/dS
// at the block end, the forward was
//   Delta = U - W S0^T,  O = Qt S0^T + P Delta,  S_end = e^(G_last) S0 + Delta^T Kt,
// and its gradient, taken back step by step (dO = dL/dO from the output step):
//   dDelta = P^T dO + Kt dS^T
//   dS0    = e^(G_last) dS + dO^T Qt - dDelta^T W              (the reverse scan)
//   dQ     = diag(E) dO S0 + dQK K,     dQK = (dO Delta^T) o Gam,  Gam_rj = [j <= r] e^(G_r - G_j)
//   dK     = dQK^T Q + diag(e^(G_last - G)) Delta dS + diag(beta E) dKb + (dA + dA^T) K
//   dKb    = T^T dW,  dW = -dDelta S0;   dVb = T^T dDelta,  dV = diag(beta) dVb
//   dL     = -(dKb W^T + dVb U^T) o [j < r]   (from d(I + L)^-1 = -T dL T, with W^T = Kb^T T^T)
//   dA     = diag(beta) dL o Gam,  A = K K^T
//   dbeta  = E rowsum(dKb o K) + rowsum(dVb o V) + rowsum(dL o Gam o A)
//   dG     = rowsum(dP o P) - colsum(dP o P) + rowsum(dLL) - colsum(dLL) - rowsum(dKd o Kt)
//            + E (rowsum(dO S0 o Q) + beta rowsum(dKb o K)),  dLL = diag(beta) dL o Gam o A,
//   and d log alpha = the reverse cumulative sum of dG over the block, plus
//   dG_last = e^(G_last) <dS, S0> + sum(dKd o Kt) on every token.
//
// Kernels:
//   gdn_bwd_scan_kernel  the reverse scan of dS over segments of blocks, in the transposed form
//                        dS^T <- e^(G_last) dS^T + Qt^T dO - W^T dDelta (state dS^T in TMEM, fp32):
//                        a transfer pass from zero at each segment end (segments 1 .. NS-1), then,
//                        after the combine, a final pass that writes dS^T at every block end (fp16).
//                        A segment's transfer is the forward's transposed, so the forward's P^T
//                        serves the combine.
//   gdn_bwd_grad_kernel  every block's local gradients: 16 tcgen05 products of 128 x 128 x 128,
//                        five epilogues; persistent, one CTA per SM.
#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

__device__ __forceinline__ bool warp_wait_all(uint64_t *bar, uint32_t ph, volatile AbortState *ab, int *status,
                                              uint64_t lim) {
    return __all_sync(0xffffffffu, mbar_wait_ol(bar, ph, ab, status, lim));
}

// 32 values as fp16 into row r, columns col .. col+31 (col a multiple of 32), of a 128-row panel tile
__device__ __forceinline__ void put_h32(uint8_t *tile, int r, int col, const float (&v)[32]) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        uint4 u;
        u.x = pack_half2(v[8 * k], v[8 * k + 1]);
        u.y = pack_half2(v[8 * k + 2], v[8 * k + 3]);
        u.z = pack_half2(v[8 * k + 4], v[8 * k + 5]);
        u.w = pack_half2(v[8 * k + 6], v[8 * k + 7]);
        *reinterpret_cast<uint4 *>(tile + tile_off(128, r, col / 8 + k)) = u;
    }
}

// 8 fp16 values (16-byte chunk c16 of row r of a 128-row panel tile) as fp32
__device__ __forceinline__ void tile_h8(const uint8_t *tile, int r, int c16, float (&f)[8]) {
    const uint4 v = *reinterpret_cast<const uint4 *>(tile + tile_off(128, r, c16));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 x = unpack_half2(w[e]);
        f[2 * e] = x.x;
        f[2 * e + 1] = x.y;
    }
}
// A warp's 32 x 32 block (lane = row, v = its 32 columns) transposed in registers: afterwards lane l
// holds column l (v[k] = row k).  Five exchange stages; at stage m a lane trades the elements whose
// index differs from its own lane index in bit m with lane ^ m.
__device__ __forceinline__ void transpose32(float (&v)[32], int lane) {
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) {
        const bool b = (lane & m) != 0;
#pragma unroll
        for (int j0 = 0; j0 < 32; ++j0) {
            if (j0 & m) continue;
            const int j1 = j0 | m;
            const float send = b ? v[j0] : v[j1];
            const float recv = __shfl_xor_sync(0xffffffffu, send, m);
            if (b) v[j0] = recv;
            else v[j1] = recv;
        }
    }
}
// A warp's 32 rows x 32 columns of fp32 output (lane = row) to rows row0 .. row0+31 of a [.][128]
// array, columns c0 .. c0+31: transposed first, so that each store writes one row's 128 bytes.
__device__ __forceinline__ void store_rows32(float *dst, size_t row0, int c0, float (&v)[32], int lane) {
    transpose32(v, lane);
#pragma unroll
    for (int k = 0; k < 32; ++k) dst[(row0 + k) * 128 + c0 + lane] = v[k];
}

// 32 fp32 values to global memory (16-byte aligned)
__device__ __forceinline__ void st_f32(float *dst, const float (&v)[32], float s) {
#pragma unroll
    for (int k = 0; k < 8; ++k)
        reinterpret_cast<float4 *>(dst)[k] = make_float4(s * v[4 * k], s * v[4 * k + 1], s * v[4 * k + 2], s * v[4 * k + 3]);
}

// Column sums of a warp's 32 x 32 block (lane = row, v = the row's 32 columns): a reduce-scatter
// by halving exchanges; lane l ends with the sum of column l.
__device__ __forceinline__ float colsum32(float (&v)[32], int lane) {
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) {
        const bool up = (lane & m) != 0;
#pragma unroll
        for (int i = 0; i < m; ++i) {
            const float send = up ? v[i] : v[i + m];
            const float keep = up ? v[i + m] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
        }
    }
    return v[0];
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
}

// Operand descriptors of a 128 x 128 fp16 panel tile at byte offset `base` of shared memory, for
// the 16-wide K step kk: K along the tile's columns (K-major) or along its rows (MN-major).
__device__ __forceinline__ uint64_t kdesc(uint32_t base, int kk) {
    return sdesc_sw128(base + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
}
__device__ __forceinline__ uint64_t mdesc(uint32_t base, int kk) { return sdesc_sw128(base + kk * 2048, 16384, 1024); }

// D (+)= A B over K = 128: eight 16-wide steps; accumulate = false overwrites D on the first step.
// A step's descriptor is the first one with the step's byte offset / 16 added to its address field
// (no carry out of it: shared-memory addresses stay below 256 KB).
__device__ __forceinline__ void gemm128(uint32_t d, uint32_t a, bool a_mn, uint32_t b, bool b_mn, bool accumulate) {
    const uint32_t id = idesc_f16_f32(128, 128, a_mn, b_mn);
    const uint64_t da = a_mn ? mdesc(a, 0) : kdesc(a, 0), db = b_mn ? mdesc(b, 0) : kdesc(b, 0);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
        const uint32_t ka = a_mn ? kk * 2048 : (kk >> 2) * 16384 + (kk & 3) * 32;
        const uint32_t kb = b_mn ? kk * 2048 : (kk >> 2) * 16384 + (kk & 3) * 32;
        umma_f16(d, da + (ka >> 4), db + (kb >> 4), id, (accumulate || kk > 0) ? 1u : 0u);
    }
}

// ============================================================ reverse scan of dS
namespace bs {
constexpr uint32_t OFF_P = 0, OFF_DO = 32768, OFF_KT = 65536, OFF_QT = 98304, OFF_W = 131072;
constexpr uint32_t OFF_S = 163840;  // dS^T fp16, rows d_k, columns d_v (MN-major B of Kt dS^T)
constexpr uint32_t OFF_R = 196608;  // -dDelta fp16, rows token, columns d_v (MN-major B of W^T (-dDelta))
constexpr uint32_t OFF_BAR = 229376;
enum { FULL_PK = 0, FULL_DQW, MMA_R, MMA_X, CONS_R, CONS_S, NBAR };
constexpr uint32_t SMEM_BYTES = OFF_BAR + NBAR * 8 + 16 + 1024;
constexpr uint32_t TM_S = 0, TM_R = 128, TM_X = 256;
constexpr int kThreads = 160;  // warps 0-3: TMEM lanes (state rows, dDelta rows); warp 4: loads and MMAs
}  // namespace bs

template <bool kFinal>
__global__ void __launch_bounds__(bs::kThreads, 1)
    gdn_bwd_scan_kernel(const BwdTcParams p, const __grid_constant__ CUtensorMap tmAqk,
                        const __grid_constant__ CUtensorMap tmDO, const __grid_constant__ CUtensorMap tmKt,
                        const __grid_constant__ CUtensorMap tmQt, const __grid_constant__ CUtensorMap tmW) {
    using namespace bs;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + NBAR);
    AbortState *ab = reinterpret_cast<AbortState *>(tmem_slot + 1);

    const int seg = kFinal ? static_cast<int>(blockIdx.x) : static_cast<int>(blockIdx.x) + 1;
    const int bh = blockIdx.y;
    const int c0 = seg * p.Ls, c1 = min(c0 + p.Ls, p.NB);
    const int n = c1 - c0;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint64_t lim = p.wait_limit_ns;

    if (tid == 0) {
        for (int i = 0; i < NBAR; ++i) mbar_init(&bars[i], (i == CONS_R || i == CONS_S) ? 4 : 1);
        ab->flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    pdl_launch_dependents();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_wait();  // the previous kernel's outputs (dO, the segment-end gradients) are complete

    if (warp == 4) {
        if (lane == 0 && n > 0) {
            const int rowbase = bh * p.Tp;
            int started[CONS_R] = {};  // phases started on FULL_PK, FULL_DQW, MMA_R, MMA_X (for the drain)
            auto load2 = [&](uint32_t off, const CUtensorMap *m, uint64_t *bar, int c) {
                tma_load_2d(sm + off, m, bar, 0, rowbase + c * kBlk);
                tma_load_2d(sm + off + 16384, m, bar, 64, rowbase + c * kBlk);
            };
            auto load_pk = [&](int c) {
                ++started[FULL_PK];
                mbar_arrive_expect_tx(&bars[FULL_PK], 65536);
                load2(OFF_P, &tmAqk, &bars[FULL_PK], c);
                load2(OFF_KT, &tmKt, &bars[FULL_PK], c);
            };
            auto load_dqw = [&](int c) {
                ++started[FULL_DQW];
                mbar_arrive_expect_tx(&bars[FULL_DQW], 98304);
                load2(OFF_DO, &tmDO, &bars[FULL_DQW], c);
                load2(OFF_QT, &tmQt, &bars[FULL_DQW], c);
                load2(OFF_W, &tmW, &bars[FULL_DQW], c);
            };
            load_pk(c1 - 1);
            load_dqw(c1 - 1);
            bool ok = true;
            for (int k = 0; ok && k < n; ++k) {
                const int c = c1 - 1 - k;
                const uint32_t ph = k & 1;
                if (c - 2 >= c0) {  // the tiles of block c-2 into L2 ahead of their loads
                    const int y2 = rowbase + (c - 2) * kBlk;
                    for (int hf = 0; hf < 2; ++hf) {
                        tma_prefetch_2d(&tmAqk, hf * 64, y2);
                        tma_prefetch_2d(&tmKt, hf * 64, y2);
                        tma_prefetch_2d(&tmDO, hf * 64, y2);
                        tma_prefetch_2d(&tmQt, hf * 64, y2);
                        tma_prefetch_2d(&tmW, hf * 64, y2);
                    }
                }
                ok = mbar_wait(&bars[FULL_PK], ph, ab, p.status, lim) && mbar_wait(&bars[FULL_DQW], ph, ab, p.status, lim);
                if (!ok) break;
                tc_fence_after();
                // dDelta = P^T dO  (A = P read MN-major: M = token i, K = token r; B = dO MN-major)
                gemm128(tmem + TM_R, sbase + OFF_P, true, sbase + OFF_DO, true, false);
                ok = mbar_wait(&bars[CONS_S], ph, ab, p.status, lim);  // dS^T copy ready, X read out
                if (!ok) break;
                tc_fence_after();
                // dDelta += Kt dS^T  (A = Kt K-major; B = dS^T MN-major: K = d_k, N = d_v)
                gemm128(tmem + TM_R, sbase + OFF_KT, false, sbase + OFF_S, true, true);
                umma_commit(&bars[MMA_R]);
                ++started[MMA_R];
                // X = Qt^T dO  (A = Qt MN-major: M = d_k, K = token)
                gemm128(tmem + TM_X, sbase + OFF_QT, true, sbase + OFF_DO, true, false);
                ok = mbar_wait(&bars[MMA_R], ph, ab, p.status, lim);
                if (!ok) break;
                if (k + 1 < n) load_pk(c - 1);
                ok = mbar_wait(&bars[CONS_R], ph, ab, p.status, lim);  // -dDelta in the R tile
                if (!ok) break;
                tc_fence_after();
                // X += W^T (-dDelta)  (A = W MN-major: M = d_k, K = token; B = -dDelta MN-major)
                gemm128(tmem + TM_X, sbase + OFF_W, true, sbase + OFF_R, true, true);
                umma_commit(&bars[MMA_X]);
                ++started[MMA_X];
                ok = mbar_wait(&bars[MMA_X], ph, ab, p.status, lim);
                if (!ok) break;
                if (k + 1 < n) load_dqw(c - 1);
            }
            // loads and products still in flight (after an abort) complete before shared memory and
            // TMEM go away; immediate when everything has completed
#pragma unroll
            for (int kb = 0; kb < CONS_R; ++kb)
                if (started[kb] > 0) mbar_wait_drain(&bars[kb], (started[kb] - 1) & 1, lim);
        }
    } else if (n > 0) {
        // ---------------------------------------------------------------- TMEM lanes
        const int r = tid;  // row of dS^T (d_k) in TM_S / TM_X, token row of dDelta in TM_R
        const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
        // dS^T at the segment end: from the combine, or zero (the sequence end; a transfer pass)
        const float *src = (kFinal && seg < p.NS - 1)
                               ? p.dSend + ((static_cast<size_t>(bh) * p.NS + seg) * 128 + r) * 128
                               : nullptr;
        __half *g0 = kFinal ? p.dSb + (static_cast<size_t>(bh) * p.Tp + static_cast<size_t>(c1 - 1) * kBlk + r) * 128
                            : nullptr;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
            float v[32];
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
                const float4 x = src ? *reinterpret_cast<const float4 *>(src + ch * 32 + e) : make_float4(0.f, 0.f, 0.f, 0.f);
                v[e] = x.x; v[e + 1] = x.y; v[e + 2] = x.z; v[e + 3] = x.w;
            }
            tmem_st32(tmem + lane_base + TM_S + ch * 32, v);
            put_h32(sm + OFF_S, r, ch * 32, v);
            if (g0) {
                float w[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) w[e] = v[e];
                uint4 *gd = reinterpret_cast<uint4 *>(g0 + ch * 32);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    gd[k] = make_uint4(pack_half2(w[8 * k], w[8 * k + 1]), pack_half2(w[8 * k + 2], w[8 * k + 3]),
                                       pack_half2(w[8 * k + 4], w[8 * k + 5]), pack_half2(w[8 * k + 6], w[8 * k + 7]));
            }
        }
        tmem_st_wait();
        fence_proxy_async();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[CONS_S]);

        const float *Gbh = p.G + static_cast<size_t>(bh) * p.Tp;
        bool done = true;
        for (int k = 0; k < n; ++k) {
            done = false;
            const int c = c1 - 1 - k;
            const uint32_t ph = k & 1;
            const float gC = __expf(fminf(Gbh[c * kBlk + kBlk - 1], 0.0f));
            if (!warp_wait_all(&bars[MMA_R], ph, ab, p.status, lim)) break;
            tc_fence_after();
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {  // -dDelta, token row r
                float x[32];
                tmem_ld32(tmem + lane_base + TM_R + ch * 32, x);
#pragma unroll
                for (int e = 0; e < 32; ++e) x[e] = -x[e];
                put_h32(sm + OFF_R, r, ch * 32, x);
            }
            fence_proxy_async();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[CONS_R]);
            if (!warp_wait_all(&bars[MMA_X], ph, ab, p.status, lim)) break;
            tc_fence_after();
            // dS^T row r <- e^(G_last) dS^T row r + X row r: the gradient at the start of block c,
            // which is the end of block c - 1
            __half *gs = (kFinal && c - 1 >= c0)
                             ? p.dSb + (static_cast<size_t>(bh) * p.Tp + static_cast<size_t>(c - 1) * kBlk + r) * 128
                             : nullptr;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                float x[32], sv[32];
                tmem_ld32(tmem + lane_base + TM_X + ch * 32, x);
                tmem_ld32(tmem + lane_base + TM_S + ch * 32, sv);
#pragma unroll
                for (int e = 0; e < 32; ++e) sv[e] = fmaf(gC, sv[e], x[e]);
                tmem_st32(tmem + lane_base + TM_S + ch * 32, sv);
                put_h32(sm + OFF_S, r, ch * 32, sv);
                if (gs) {
                    uint4 *gd = reinterpret_cast<uint4 *>(gs + ch * 32);
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        gd[q] = make_uint4(pack_half2(sv[8 * q], sv[8 * q + 1]), pack_half2(sv[8 * q + 2], sv[8 * q + 3]),
                                           pack_half2(sv[8 * q + 4], sv[8 * q + 5]), pack_half2(sv[8 * q + 6], sv[8 * q + 7]));
                }
            }
            tmem_st_wait();
            fence_proxy_async();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[CONS_S]);
            done = true;
        }
        if (!kFinal && done) {  // the segment's local dS^T (fp32) for the combine
            tc_fence_after();
            float *dst = p.dSloc + ((static_cast<size_t>(bh) * p.NS + seg) * 128 + r) * 128;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                float sv[32];
                tmem_ld32(tmem + lane_base + TM_S + ch * 32, sv);
                st_f32(dst + ch * 32, sv, 1.0f);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

// ============================================================ local gradients of every block
namespace bg {
// 16 warps: TMEM lane quarter w & 3, 32-column quarter w >> 2 of every accumulator.  Thread 0 also
// issues the TMA loads and the tensor-core products, each phase's after the barrier that ends the
// previous epilogue (so there is no separate producer warp, and 128 registers per thread).
constexpr int kThreads = 512;
constexpr uint32_t SLOT = 32768;                 // six 128 x 128 fp16 tile slots
constexpr uint32_t OFF_G = 6 * SLOT;             // fp32 [128]: G of the block
constexpr uint32_t OFF_COL = OFF_G + 512;        // fp32 [4][128]: column sums over each lane quarter's rows
constexpr uint32_t OFF_X = OFF_COL + 2048;       // fp32 [3][4][128]: row partials of column quarters 1-3
constexpr uint32_t OFF_WS = OFF_X + 6144;        // fp32 [16][2] per-warp sums, [4] suffix-scan totals
constexpr uint32_t OFF_CNT = OFF_WS + 256;       // int [6] loads per slot, [11] phases per barrier (thread 0)
constexpr uint32_t OFF_BAR = OFF_CNT + 128;
enum { FULL0 = 0, MMA_A = 6, MMA_B, MMA_C, MMA_D, MMA_E, NBAR };
constexpr uint32_t SMEM_BYTES = OFF_BAR + NBAR * 8 + 16 + 1024;
constexpr uint32_t TM0 = 0, TM1 = 128, TM2 = 256, TM3 = 384;
}  // namespace bg

// 32 fp16 values (64 contiguous bytes of global memory) kept packed, for use after a wait
__device__ __forceinline__ void pf_h32(const __half *src, uint4 (&u)[4]) {
    const uint4 *s4 = reinterpret_cast<const uint4 *>(src);
#pragma unroll
    for (int k = 0; k < 4; ++k) u[k] = s4[k];
}
// element e (a compile-time index) of a packed 32-value row
__device__ __forceinline__ float hget(const uint4 (&u)[4], int e) {
    const uint4 v = u[e >> 3];
    const int wi = (e & 7) >> 1;
    const uint32_t w = wi == 0 ? v.x : (wi == 1 ? v.y : (wi == 2 ? v.z : v.w));
    const float2 f = unpack_half2(w);
    return (e & 1) ? f.y : f.x;
}

// Slot use per block (s0 .. s5), tile loaded by TMA or written by the epilogue (E*):
//   phase A: S0^T s0, W s1, dO s2, P s3, Kt s4, dS^T s5   -> A3 dO S0 (TM2), A1 W S0^T (TM0),
//                                                           A2 P^T dO + Kt dS^T (TM1)
//   EA: Delta -> s3, dDelta -> s4, TM2 *= E;  then K -> s1
//   phase B: B1 dO Delta^T (TM0), B2 Delta dS (TM3), B3 dDelta S0 (TM1)
//   EB: dQK -> s3, dW -> s5, TM3 = e^(G_last - G) o TM3;  Q -> s0, T -> s2
//   phase C: C1 TM2 += dQK K, C2 TM3 += dQK^T Q, C3 T^T dW (TM0), C4 T^T dDelta (TM1)
//   EC: dQ out, dKb -> s3, dVb -> s4, TM3 += diag(beta E) dKb, dV out;  W -> s0, U -> s2
//   phase D: D1 dKb W^T + dVb U^T (TM0), D2 K K^T (TM1)
//   ED: dA -> s5;  the next block's S0^T -> s0, dO -> s2, P -> s3, Kt -> s4
//   phase E: E1 TM3 += dA K + dA^T K
//   EE: dK out, row and column sums, d log alpha, dbeta;  the next block's W -> s1, dS^T -> s5
__global__ void __launch_bounds__(bg::kThreads, 1)
    gdn_bwd_grad_kernel(const BwdTcParams p, const __grid_constant__ BwdTcMaps m) {
    using namespace bg;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + NBAR);
    AbortState *ab = reinterpret_cast<AbortState *>(tmem_slot + 1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint64_t lim = p.wait_limit_ns;
    const int total = p.BH * p.NB;

    if (tid == 0) {
        for (int i = 0; i < NBAR; ++i) mbar_init(&bars[i], 1);
        ab->flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    pdl_launch_dependents();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_wait();  // dS^T at every block end is complete

    // thread 0's loads and products; its counters live in shared memory, not in every thread's registers
    int *nld = reinterpret_cast<int *>(sm + OFF_CNT);  // loads issued into each slot
    int *started = nld + 6;                            // phases started on every barrier (for the drain)
    if (tid == 0)
        for (int k = 0; k < 6 + NBAR; ++k) nld[k] = 0;
    auto load = [&](int slot, const CUtensorMap *map, int w) {
        const int y = (w / p.NB) * p.Tp + (w % p.NB) * kBlk;
        uint64_t *bar = &bars[FULL0 + slot];
        mbar_arrive_expect_tx(bar, SLOT);
        tma_load_2d(sm + slot * SLOT, map, bar, 0, y);
        tma_load_2d(sm + slot * SLOT + 16384, map, bar, 64, y);
        ++nld[slot];
        ++started[FULL0 + slot];
    };
    auto ready = [&](int slot) { return mbar_wait(&bars[FULL0 + slot], (nld[slot] - 1) & 1, ab, p.status, lim); };
    auto commit = [&](int b) {
        umma_commit(&bars[b]);
        ++started[b];
    };
    // the slots' addresses, re-formed wherever products are issued (an opaque copy of the base) so that
    // the descriptors of the block's 16 products are not all kept live across the loop
    uint32_t s0, s1, s2, s3, s4, s5;
    auto slots = [&]() {
        uint32_t b;
        asm volatile("mov.b32 %0, %1;" : "=r"(b) : "r"(sbase));
        s0 = b; s1 = b + SLOT; s2 = b + 2 * SLOT; s3 = b + 3 * SLOT; s4 = b + 4 * SLOT; s5 = b + 5 * SLOT;
    };

    const int q = warp & 3, cq = warp >> 2;
    const int r = q * 32 + lane;  // the block row (token) this thread owns, columns cb .. cb + 31
    const int cb = cq * 32;
    const uint32_t lb = tmem + (static_cast<uint32_t>(q * 32) << 16) + cb;
    float *sG = reinterpret_cast<float *>(sm + OFF_G);
    float *colpart = reinterpret_cast<float *>(sm + OFF_COL);
    float *xch = reinterpret_cast<float *>(sm + OFF_X);
    float *wsum = reinterpret_cast<float *>(sm + OFF_WS);
    uint8_t *t3 = sm + 3 * SLOT, *t4 = sm + 4 * SLOT, *t5 = sm + 5 * SLOT;
    const bool issuer = tid == 0;
    // after an epilogue: its shared-memory tiles visible to the tensor cores and its TMEM accesses
    // ordered before the next products, for the issuing thread
    auto end_phase = [&]() {
        tmem_st_wait();
        fence_proxy_async();
        tc_fence_before();
        named_sync(2, kThreads);
        if (issuer) tc_fence_after();
    };

    if (issuer && blockIdx.x < total) {
        const int w = blockIdx.x;
        load(0, &m.S0, w);
        load(1, &m.W, w);
        load(2, &m.dO, w);
        load(3, &m.Aqk, w);
        load(4, &m.Kt, w);
        load(5, &m.dS, w);
    }
    for (int w = blockIdx.x, i = 0; w < total; w += gridDim.x, ++i) {
        const uint32_t ph = i & 1;
        const int wn = w + gridDim.x;
        const int bh = w / p.NB, c = w % p.NB;
        const size_t row0 = static_cast<size_t>(bh) * p.Tp + static_cast<size_t>(c) * kBlk;
        const size_t grow = row0 + r;
        const size_t gel = grow * 128 + cb;  // element offset of this thread's columns in [BH][Tp][128]
        const float Gr = p.G[grow], be = p.beta[grow], gL = p.G[row0 + kBlk - 1];
        const float Er = __expf(Gr), fr = __expf(fminf(gL - Gr, 0.0f)), eC = __expf(gL);
        if (cq == 0) sG[r] = Gr;
        float dG = 0.0f, dbeta = 0.0f, dE = 0.0f, sdot = 0.0f, sdgc = 0.0f;
        uint4 pa[4], pb[4];
        pf_h32(p.U + gel, pa);
        pf_h32(p.Q + gel, pb);

        // ---- phase A (the previous block's epilogues have read TM0-TM2)
        if (issuer && ready(0) && ready(1) && ready(2) && ready(3) && ready(4) && ready(5)) {
            tc_fence_after();
            slots();
            gemm128(tmem + TM2, s2, false, s0, false, false);  // A3: dO S0 (B = S0^T read K-major)
            gemm128(tmem + TM0, s1, false, s0, true, false);   // A1: W S0^T (B = S0^T MN-major)
            gemm128(tmem + TM1, s3, true, s2, true, false);    // A2: P^T dO
            gemm128(tmem + TM1, s4, false, s5, true, true);    //     + Kt dS^T
            commit(MMA_A);
        }
        // ---- EA: Delta = U - W S0^T -> s3;  dDelta -> s4;  TM2 = E o dO S0, rowsum(dO S0 o Q);  <dS, S0>
        //      (U and Q rows fetched before the wait; S0^T and dS^T rows from their tiles)
        bool ok = warp_wait_all(&bars[MMA_A], ph, ab, p.status, lim) &&
                  warp_wait_all(&bars[FULL0 + 0], ph, ab, p.status, lim) &&  // S0^T: load 3i of slot 0
                  warp_wait_all(&bars[FULL0 + 5], ph, ab, p.status, lim);    // dS^T: load i of slot 5
        if (!group_all(1, kThreads, ok)) break;
        tc_fence_after();
        {
            float x[32];
            tmem_ld32(lb + TM0, x);
#pragma unroll
            for (int e = 0; e < 32; ++e) x[e] = hget(pa, e) - x[e];
            put_h32(t3, r, cb, x);
            tmem_ld32(lb + TM1, x);
            put_h32(t4, r, cb, x);
            tmem_ld32(lb + TM2, x);
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                dE = fmaf(x[e], hget(pb, e), dE);
                x[e] *= Er;
            }
            tmem_st32(lb + TM2, x);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                float d8[8], s8[8];
                tile_h8(sm + 5 * SLOT, r, cb / 8 + k, d8);
                tile_h8(sm, r, cb / 8 + k, s8);
#pragma unroll
                for (int e = 0; e < 8; ++e) sdot = fmaf(d8[e], s8[e], sdot);
            }
        }
        pf_h32(p.Aqk + gel, pa);  // the P row EB reads, fetched while the products of phase B run
        end_phase();
        if (issuer) {  // ---- phase B (TM3 was read in the previous block's EE)
            slots();
            load(1, &m.K, w);
            gemm128(tmem + TM0, s2, false, s3, false, false);  // B1: dO Delta^T
            gemm128(tmem + TM3, s3, false, s5, false, false);  // B2: Delta dS (B = dS^T read K-major)
            gemm128(tmem + TM1, s4, false, s0, false, false);  // B3: dDelta S0
            commit(MMA_B);
        }

        // ---- EB: TM3 = e^(G_last - G) o dKd, rowsum(dKd o Kt) (= e^(G_last - G_r) rowsum(dKd o K), K from
        //      its tile: load 2i + 1 of slot 1);  dW = -dDelta S0 -> s5;  dQK = dP o Gam -> s3, rowsum /
        //      colsum of dP o P
        ok = warp_wait_all(&bars[MMA_B], ph, ab, p.status, lim) && warp_wait_all(&bars[FULL0 + 1], 1, ab, p.status, lim);
        if (!group_all(1, kThreads, ok)) break;
        tc_fence_after();
        if (issuer) {  // S0^T and dO have their last readers behind them
            load(0, &m.Q, w);
            load(2, &m.T, w);
        }
        {
            float x[32], v[32];
            float t = 0.0f;
            tmem_ld32(lb + TM3, x);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                float k8[8];
                tile_h8(sm + SLOT, r, cb / 8 + k, k8);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    t = fmaf(x[8 * k + e], k8[e], t);
                    x[8 * k + e] *= fr;
                }
            }
            tmem_st32(lb + TM3, x);
            tmem_ld32(lb + TM1, x);
#pragma unroll
            for (int e = 0; e < 32; ++e) x[e] = -x[e];
            put_h32(t5, r, cb, x);
            float rs = 0.0f;
            tmem_ld32(lb + TM0, x);
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const int j = cb + e;
                const float dpp = x[e] * hget(pa, e);
                v[e] = dpp;
                rs += dpp;
                x[e] = (j <= r) ? x[e] * __expf(Gr - sG[j]) : 0.0f;
            }
            put_h32(t3, r, cb, x);
            colpart[q * 128 + cb + lane] = colsum32(v, lane);
            t *= fr;
            dG += rs - t;
            sdgc += t;
        }
        pf_h32(p.V + gel, pa);  // the V row EC reads
        end_phase();
        if (issuer && ready(0) && ready(1) && ready(2)) {  // ---- phase C
            slots();
            gemm128(tmem + TM2, s3, false, s1, true, true);    // C1: dQ += dQK K
            gemm128(tmem + TM3, s3, true, s0, true, true);     // C2: dK += dQK^T Q
            gemm128(tmem + TM0, s2, true, s5, true, false);    // C3: dKb = T^T dW
            gemm128(tmem + TM1, s2, true, s4, true, false);    // C4: dVb = T^T dDelta
            commit(MMA_C);
        }

        // ---- EC: dQ out;  dKb -> s3, TM3 += diag(beta E) dKb, rowsum(dKb o K);  dVb -> s4,
        //      dv^ = beta dVb out, rowsum(dVb o V)
        if (!group_all(1, kThreads, warp_wait_all(&bars[MMA_C], ph, ab, p.status, lim))) break;
        tc_fence_after();
        if (issuer) {  // Q and T have their last readers behind them
            load(0, &m.W, w);
            load(2, &m.U, w);
        }
        {
            float x[32], u[32];
            float tk = 0.0f, tv = 0.0f;
            tmem_ld32(lb + TM2, x);
            store_rows32(p.dqh, row0 + q * 32, cb, x, lane);
            tmem_ld32(lb + TM0, x);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                float k8[8];
                tile_h8(sm + SLOT, r, cb / 8 + k, k8);
#pragma unroll
                for (int e = 0; e < 8; ++e) tk = fmaf(x[8 * k + e], k8[e], tk);
            }
            tmem_ld32(lb + TM3, u);
#pragma unroll
            for (int e = 0; e < 32; ++e) u[e] = fmaf(be * Er, x[e], u[e]);
            tmem_st32(lb + TM3, u);
            put_h32(t3, r, cb, x);
            tmem_ld32(lb + TM1, x);
#pragma unroll
            for (int e = 0; e < 32; ++e) tv = fmaf(x[e], hget(pa, e), tv);
            put_h32(t4, r, cb, x);
#pragma unroll
            for (int e = 0; e < 32; ++e) x[e] *= be;
            store_rows32(p.dvh, row0 + q * 32, cb, x, lane);
            dbeta = fmaf(Er, tk, dbeta) + tv;
            dE = fmaf(be, tk, dE);
        }
        end_phase();
        if (issuer && ready(0) && ready(2)) {  // ---- phase D
            slots();
            gemm128(tmem + TM0, s3, false, s0, false, false);  // D1: dKb W^T
            gemm128(tmem + TM0, s4, false, s2, false, true);   //     + dVb U^T
            gemm128(tmem + TM1, s1, false, s1, false, false);  // D2: K K^T
            commit(MMA_D);
        }

        // ---- ED: dL = -(dKb W^T + dVb U^T) below the diagonal, A = K K^T: dA = beta dL o Gam -> s5,
        //      rowsum(dL o Gam o A) into dbeta, rowsum / colsum of dLL = beta dL o Gam o A
        if (!group_all(1, kThreads, warp_wait_all(&bars[MMA_D], ph, ab, p.status, lim))) break;
        tc_fence_after();
        if (issuer && wn < total) {  // the next block's tiles into the slots phase D has freed
            const int yn = (wn / p.NB) * p.Tp + (wn % p.NB) * kBlk;
            for (int hf = 0; hf < 2; ++hf) {  // and, into L2, the rows its epilogues read from global memory
                tma_prefetch_2d(&m.U, hf * 64, yn);  // and the two tiles loaded after this block's last products
                tma_prefetch_2d(&m.Q, hf * 64, yn);
                tma_prefetch_2d(&m.V, hf * 64, yn);
                tma_prefetch_2d(&m.W, hf * 64, yn);
                tma_prefetch_2d(&m.dS, hf * 64, yn);
            }
            load(0, &m.S0, wn);
            load(2, &m.dO, wn);
            load(3, &m.Aqk, wn);
            load(4, &m.Kt, wn);
        }
        {
            float mv[32], a[32];
            float rs = 0.0f, db = 0.0f;
            tmem_ld32(lb + TM0, mv);
            tmem_ld32(lb + TM1, a);
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const int j = cb + e;
                if (j < r) {
                    const float gs = __expf(Gr - sG[j]);
                    const float dl = -mv[e];
                    const float dlga = dl * gs * a[e];
                    db += dlga;
                    a[e] = be * dlga;  // dLL
                    rs += a[e];
                    mv[e] = be * dl * gs;  // dA
                } else {
                    a[e] = 0.0f;
                    mv[e] = 0.0f;
                }
            }
            put_h32(t5, r, cb, mv);
            colpart[q * 128 + cb + lane] += colsum32(a, lane);
            dbeta += db;
            dG += rs;
        }
        end_phase();
        if (issuer) {  // ---- phase E
            slots();
            gemm128(tmem + TM3, s5, false, s1, true, true);    // E1: dK += dA K
            gemm128(tmem + TM3, s5, true, s1, true, true);     //     + dA^T K
            commit(MMA_E);
        }

        // ---- EE: dk^ out; the row sums of the four column quarters, the column sums, d log alpha
        if (!group_all(1, kThreads, warp_wait_all(&bars[MMA_E], ph, ab, p.status, lim))) break;
        tc_fence_after();
        if (issuer && wn < total) {  // K and dA have their last readers behind them
            load(1, &m.W, wn);
            load(5, &m.dS, wn);
        }
        {
            float x[32];
            tmem_ld32(lb + TM3, x);
            store_rows32(p.dkh, row0 + q * 32, cb, x, lane);
        }
        if (cq > 0) {
            xch[(0 * 4 + cq) * 128 + r] = dG;
            xch[(1 * 4 + cq) * 128 + r] = dbeta;
            xch[(2 * 4 + cq) * 128 + r] = dE;
        }
        sdot = warp_sum(sdot);
        sdgc = warp_sum(sdgc);
        if (lane == 0) {
            wsum[2 * warp] = sdot;
            wsum[2 * warp + 1] = sdgc;
        }
        tc_fence_before();
        named_sync(2, kThreads);
        if (cq == 0) {
#pragma unroll
            for (int k = 1; k < 4; ++k) {
                dG += xch[(0 * 4 + k) * 128 + r];
                dbeta += xch[(1 * 4 + k) * 128 + r];
                dE += xch[(2 * 4 + k) * 128 + r];
            }
            dG -= colpart[r] + colpart[128 + r] + colpart[256 + r] + colpart[384 + r];
            dG = fmaf(Er, dE, dG);
            float sd = 0.0f, sgc = 0.0f;
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                sd += wsum[2 * k];
                sgc += wsum[2 * k + 1];
            }
            const float dgC = fmaf(eC, sd, sgc);
            // d log alpha_r = sum_{s >= r} dG_s (+ dG_last's share on every token)
            float sc = dG;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float nb = __shfl_down_sync(0xffffffffu, sc, off);
                if (lane + off < 32) sc += nb;
            }
            if (lane == 0) wsum[32 + q] = sc;
            named_sync(3, 128);
            for (int q2 = q + 1; q2 < 4; ++q2) sc += wsum[32 + q2];
            p.dla[grow] = sc + dgC;
            p.dbeta[grow] = dbeta;
        }
    }
    if (issuer) {
        // loads and products still in flight (after an abort) complete before shared memory and TMEM go
        // away; immediate when everything has completed
#pragma unroll
        for (int kb = 0; kb < NBAR; ++kb)
            if (started[kb] > 0) mbar_wait_drain(&bars[kb], (started[kb] - 1) & 1, lim);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace

cudaError_t launch_bwd_scan(const BwdTcParams &p, bool final_pass, const CUtensorMap &tmAqk,
                            const CUtensorMap &tmDO, const CUtensorMap &tmKt, const CUtensorMap &tmQt,
                            const CUtensorMap &tmW, cudaStream_t s, bool pdl) {
    const int nseg = final_pass ? p.NS : p.NS - 1;
    if (nseg < 1) return cudaSuccess;
    const dim3 grid(nseg, p.BH);
    if (final_pass) {
        static SmemOnce once;
        cudaError_t e = raise_smem_once(once, gdn_bwd_scan_kernel<true>, static_cast<int>(bs::SMEM_BYTES));
        if (e != cudaSuccess) return e;
        return launch_k(gdn_bwd_scan_kernel<true>, grid, dim3(bs::kThreads), bs::SMEM_BYTES, s, pdl, p, tmAqk, tmDO,
                        tmKt, tmQt, tmW);
    }
    static SmemOnce once;
    cudaError_t e = raise_smem_once(once, gdn_bwd_scan_kernel<false>, static_cast<int>(bs::SMEM_BYTES));
    if (e != cudaSuccess) return e;
    return launch_k(gdn_bwd_scan_kernel<false>, grid, dim3(bs::kThreads), bs::SMEM_BYTES, s, pdl, p, tmAqk, tmDO, tmKt,
                    tmQt, tmW);
}

cudaError_t launch_bwd_grad(const BwdTcParams &p, const BwdTcMaps &m, cudaStream_t s, bool pdl) {
    static SmemOnce once;
    cudaError_t e = raise_smem_once(once, gdn_bwd_grad_kernel, static_cast<int>(bg::SMEM_BYTES));
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return cudaErrorInvalidDevice;
    const long long total = static_cast<long long>(p.BH) * p.NB;
    if (total < 1) return cudaSuccess;
    const dim3 grid(static_cast<unsigned>(total < sms ? total : sms));
    return launch_k(gdn_bwd_grad_kernel, grid, dim3(bg::kThreads), bg::SMEM_BYTES, s, pdl, p, m);
}

}  // namespace gdn
