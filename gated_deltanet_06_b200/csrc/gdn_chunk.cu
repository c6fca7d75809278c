// gdn_chunk.cu -- the intra-block UT (WY) transform of the gated delta rule
// (reference [57] on the VMonarch page) on 5th-generation tensor cores.  One
// CTA handles one 128-token block of one (b, h):
//
//   A_kk = K K^T,  QK = Q K^T             tcgen05, fp16 x fp16 -> fp32 in TMEM
//   L_rj = beta_r exp(G_r - G_j) A_kk,rj  for j < r (decay-masked strict tril)
//   T    = (I + L)^-1                     two 64x64 forward substitutions in
//                                         shared memory (fp32, one column per
//                                         thread), merged on tcgen05 through
//                                         P = L_21 T_1 and T_21^T = -P^T T_2^T
//   W    = T diag(beta e^G) K,  U = T diag(beta) V      tcgen05
//   Kt   = diag(e^(G_last - G)) K,  Qt = diag(e^G) Q,
//   Aqk  = [i <= r] e^(G_r - G_i) QK_ri
//
// and stores W, U, Kt, Qt, Aqk (fp16) for the inter-block scan with TMA bulk
// stores.  Only exponentials of non-positive differences of the cumulative
// log decay G are taken.  Two warp groups work side by side: warps 0-3 build
// L and solve for T (thread j owns column j of T), warps 4-7 build Qt and
// Aqk and Kt meanwhile, then scale the V tile and a fresh copy of the K tile
// into V~ = diag(beta) V and K~ = diag(beta e^G) K, so that T enters both
// U = T V~ and W = T K~ unscaled and its operand is built once.  Every
// operand the threads build is written in the 128B-swizzled layout the UMMA
// descriptors and the TMA read directly, one contiguous row per thread: T
// enters the W/U products transposed (MN-major), which is why the
// off-diagonal block is formed as T_21^T.  The decay factors of L and Aqk
// below the diagonal 32x32 blocks are split as e^(G_r - G_m) e^(G_m - G_j)
// (m the last row of j's group, both exponents <= 0), one exponential per
// row and per column instead of one per entry.
//
// Footprint: about 108 KB of shared memory and 256 TMEM columns, so that two
// CTAs share an SM and one's tensor and memory phases hide the other's
// thread phases.  Shared memory is reused through the block's life: the Q tile
// becomes Qt, then the staging area of Aqk, then V~, then the staging area of
// U; the K tile becomes Kt, then K~; the L blocks become the merge operands,
// then the transposed T, then the staging area of W.
#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int LD_STRIDE = 68;  // fp32 row stride of the L blocks (padded: rows written by different threads
                               // land in different banks)
// Shared-memory map (offsets from a 1024-byte aligned base).
constexpr uint32_t OFF_K = 0;              // 128x128 fp16 panel tile (TMA): K; later Kt
constexpr uint32_t OFF_QV = 32768;         // 128x128 fp16: Q -> Qt -> Aqk staging -> V (TMA) -> U staging
constexpr uint32_t OFF_LD = 65536;         // fp32 64 x 68 L_11 then 64 x 68 L_22 (34816 B); later:
constexpr uint32_t OFF_T1 = OFF_LD + 0;            //   fp16 64 x 64: T_1^T, K-major B
constexpr uint32_t OFF_T2T = OFF_LD + 8192;        //   fp16 64 x 64: T_2^T, MN-major B
constexpr uint32_t OFF_PA = OFF_LD + 16384;        //   fp16 64 rows x 128: [P | 0], MN-major A
constexpr uint32_t OFF_A = OFF_LD + 0;             //   fp16 128x128 transposed T (scaled), MN-major A; then W staging
constexpr uint32_t OFF_L21 = OFF_LD + 34816;       // fp16 64 x 64: L_21 rows, K-major
// The P = L_21 T_1 product reads a 128-row A operand starting 64 rows before L_21: its upper half
// is whatever the bytes there are, and the rows of the product it feeds are never read.
constexpr uint32_t OFF_LHA = OFF_L21 - 8192;
constexpr uint32_t OFF_G = OFF_L21 + 8192;         // fp32 [128]
constexpr uint32_t OFF_BETA = OFF_G + 512;         // fp32 [128]
constexpr uint32_t OFF_WT = OFF_BETA + 512;        // fp32 [4]: per-warp totals of the gate scan
constexpr uint32_t OFF_EC = OFF_WT + 16;           // fp32 [128]: e^(G_m - G_j), m = last row of j's 32-row group
constexpr uint32_t OFF_BAR = OFF_EC + 512;         // 4 mbarriers, tmem slot, abort flag
constexpr uint32_t SMEM_USED = OFF_BAR + 48;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // + alignment slack
static_assert(OFF_LHA % 1024 == 0 && OFF_L21 % 1024 == 0 && OFF_PA % 1024 == 0, "swizzle atoms need 1 KB alignment");
static_assert(SMEM_BYTES * 2 <= 227 * 1024, "two CTAs per SM");

constexpr uint32_t TM_AKK = 0, TM_QK = 128, TM_Y = 0, TM_D2 = 64, TM_U = 128, TM_W = 0;  // 256 columns

__device__ __forceinline__ void put8(uint8_t *tile, int rows, int r, int chunk16, const float *v) {
    uint4 u;
    u.x = pack_half2(v[0], v[1]);
    u.y = pack_half2(v[2], v[3]);
    u.z = pack_half2(v[4], v[5]);
    u.w = pack_half2(v[6], v[7]);
    *reinterpret_cast<uint4 *>(tile + tile_off(rows, r, chunk16)) = u;
}

// named barrier for one warp group (128 threads); id 1 or 2
__device__ __forceinline__ void group_sync(int id) { asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory"); }

// Transposed, column-scaled T as an MN-major A operand: row j holds T[0..127][j] * s_j.
// Thread j (warps 0-3) owns column j: T_1 / T_2 entries are in col[], the T_21 entries
// (j < 64) in TMEM lane j as -D2.
__device__ __forceinline__ void build_tT(uint8_t *dst, int j, const float (&col)[64], float s, uint32_t tD2) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        float lo[8], hi[8];
        if (j < 64) {
            float d[8];
            tmem_ld8(tD2 + c * 8, d);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                lo[e] = col[c * 8 + e] * s;
                hi[e] = -d[e] * s;
            }
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                lo[e] = 0.0f;
                hi[e] = col[c * 8 + e] * s;
            }
        }
        put8(dst, 128, j, c, lo);
        put8(dst, 128, j, 8 + c, hi);
    }
}

__global__ void __launch_bounds__(256, 2)
    gdn_chunk_kernel(const ChunkParams p, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmU,
                     const __grid_constant__ CUtensorMap tmQt, const __grid_constant__ CUtensorMap tmKt,
                     const __grid_constant__ CUtensorMap tmAqk) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    float *sG = reinterpret_cast<float *>(sm + OFF_G);
    float *sBeta = reinterpret_cast<float *>(sm + OFF_BETA);
    float *sEc = reinterpret_cast<float *>(sm + OFF_EC);
    uint64_t *bar_load = reinterpret_cast<uint64_t *>(sm + OFF_BAR);  // K and Q tiles
    uint64_t *bar_mma = bar_load + 1;
    uint64_t *bar_v = bar_load + 2;   // V tile
    uint64_t *bar_kr = bar_load + 3;  // K tile again, after Kt has been stored from it
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_load + 4);
    AbortState *ab = reinterpret_cast<AbortState *>(tmem_slot + 1);

    const int blk = blockIdx.x, bh = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5;
    const bool groupL = tid < 128;  // warps 0-3: L and T;  warps 4-7: Qt, Aqk
    const int r = tid & 127;        // TMEM lane / row (or T column) owned by this thread
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const size_t row0 = static_cast<size_t>(bh) * p.Tp + static_cast<size_t>(blk) * kBlk;
    const int y0 = static_cast<int>(row0);

    if (tid == 0) {
        mbar_init(bar_load, 1);
        mbar_init(bar_mma, 1);
        mbar_init(bar_v, 1);
        mbar_init(bar_kr, 1);
        ab->flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 256);
        tmem_relinquish();
    }
    __syncthreads();  // barrier init visible before the TMA below uses it
    if (tid == 0) {
        mbar_arrive_expect_tx(bar_load, 2u * 32768u);
        tma_load_2d(sm + OFF_K, &tmK, bar_load, 0, y0);
        tma_load_2d(sm + OFF_K + 16384, &tmK, bar_load, 64, y0);
        tma_load_2d(sm + OFF_QV, &tmQ, bar_load, 0, y0);
        tma_load_2d(sm + OFF_QV + 16384, &tmQ, bar_load, 64, y0);
    }
    if (groupL) {
        // gates of the block while the tiles land: log alpha = -exp(A_log) softplus(g + dt_bias),
        // beta = sigmoid(b), G = inclusive cumulative sum of log alpha over the block
        float *warp_tot = reinterpret_cast<float *>(sm + OFF_WT);
        const int bb = bh / p.H, hh = bh - bb * p.H;
        const int t = blk * kBlk + r;
        float la = 0.0f, be = 0.0f;
        if (t < p.T) {
            const size_t gi = (static_cast<size_t>(bb) * p.T + t) * p.H + hh;
            const float xg = p.g[gi] + p.dt_bias[hh];
            const float sp = xg > 20.0f ? xg : __logf(1.0f + __expf(xg));
            la = -__expf(p.A_log[hh]) * sp;
            be = __fdividef(1.0f, 1.0f + __expf(-p.bg[gi]));
        }
        float cs = la;
        const int lane = tid & 31;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float n = __shfl_up_sync(0xffffffffu, cs, off);
            if (lane >= off) cs += n;
        }
        if (lane == 31) warp_tot[warp] = cs;
        group_sync(1);
        for (int w = 0; w < warp; ++w) cs += warp_tot[w];
        sG[r] = cs;
        sBeta[r] = be;
        p.G[row0 + r] = cs;
        p.beta[row0 + r] = be;
        p.log_alpha[row0 + r] = la;
        group_sync(1);
        // column factors of the split decay: for j in 32-row group c and r past that group,
        // e^(G_r - G_j) = e^(G_r - G_m) e^(G_m - G_j) with m = 32c + 31, both exponents <= 0
        sEc[r] = __expf(fminf(sG[r | 31] - cs, 0.0f));
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    uint32_t mma_phase = 0;
    float col[64];
    if (tid == 0) GDN_TRACE_AT(0);
    mbar_wait(bar_load, 0, ab, p.status, p.wait_limit_ns);
    if (tid == 0) GDN_TRACE_AT(1);
    __syncthreads();
    if (ab->flag) goto teardown;

    // ---- A_kk = K K^T and Q K^T (M = N = K = 128; both operands K-major)
    if (tid == 0) {
        tc_fence_after();
        const uint32_t idesc = idesc_f16_f32(128, 128, false, false);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const uint32_t koff = (kk >> 2) * 16384 + (kk & 3) * 32;
            const uint64_t dk = sdesc_sw128(sbase + OFF_K + koff, 16, 1024);
            umma_f16(tmem + TM_AKK, dk, dk, idesc, kk > 0);
            umma_f16(tmem + TM_QK, sdesc_sw128(sbase + OFF_QV + koff, 16, 1024), dk, idesc, kk > 0);
        }
        umma_commit(bar_mma);
    }
    mbar_wait(bar_mma, mma_phase, ab, p.status, p.wait_limit_ns);
    mma_phase ^= 1;
    __syncthreads();
    if (ab->flag) goto teardown;
    tc_fence_after();

    if (groupL) {
        // ---- L row r: fp32 diagonal blocks for the solves; fp16 L_21 rows for P = L_21 T_1.
        //      Warp w owns rows 32w .. 32w+31: column group c < w lies wholly below the diagonal
        //      (split decay, no exponential per entry), c == w holds the diagonal, c > w is zero
        //      and never read.
        const float Gr = sG[r], br = sBeta[r];
        float *Ld1 = reinterpret_cast<float *>(sm + OFF_LD);
        float *Ld2 = Ld1 + 64 * LD_STRIDE;
#pragma unroll 1
        for (int c = 0; c <= warp; ++c) {
            float a[32];
            tmem_ld32(tmem + lane_base + TM_AKK + c * 32, a);
            float l[32];
            if (c < warp) {
                const float fr = br * __expf(fminf(Gr - sG[c * 32 + 31], 0.0f));
#pragma unroll
                for (int i = 0; i < 32; ++i) l[i] = fr * sEc[c * 32 + i] * a[i];
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int j = c * 32 + i;
                    l[i] = (j < r) ? br * __expf(fminf(Gr - sG[j], 0.0f)) * a[i] : 0.0f;
                }
            }
            if (c < 2) {
                if (r < 64) {
#pragma unroll
                    for (int i = 0; i < 32; i += 4)
                        *reinterpret_cast<float4 *>(Ld1 + r * LD_STRIDE + c * 32 + i) =
                            make_float4(l[i], l[i + 1], l[i + 2], l[i + 3]);
                } else {
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) put8(sm + OFF_LHA, 128, r, c * 4 + q4, &l[q4 * 8]);
                }
            } else {  // c >= 2 implies r >= 64
#pragma unroll
                for (int i = 0; i < 32; i += 4)
                    *reinterpret_cast<float4 *>(Ld2 + (r - 64) * LD_STRIDE + (c - 2) * 32 + i) =
                        make_float4(l[i], l[i + 1], l[i + 2], l[i + 3]);
            }
        }
        fence_proxy_async();
        group_sync(1);
        if (tid == 0) GDN_TRACE_AT(2);
        // ---- two 64x64 unit lower-triangular inverses, one column per thread;
        //      four independent partial sums per row keep the FMA pipe busy
        {
            const int i = r & 63;
            const float *Ld = r < 64 ? Ld1 : Ld2;
#pragma unroll
            for (int rr = 0; rr < 64; ++rr) {
                float a0 = (rr == i) ? 1.0f : 0.0f, a1 = 0.0f, a2 = 0.0f, a3 = 0.0f;
#pragma unroll
                for (int j4 = 0; j4 < rr; j4 += 4) {
                    const float4 l = *reinterpret_cast<const float4 *>(Ld + rr * LD_STRIDE + j4);
                    a0 = fmaf(-l.x, col[j4], a0);
                    if (j4 + 1 < rr) a1 = fmaf(-l.y, col[j4 + 1], a1);
                    if (j4 + 2 < rr) a2 = fmaf(-l.z, col[j4 + 2], a2);
                    if (j4 + 3 < rr) a3 = fmaf(-l.w, col[j4 + 3], a3);
                }
                col[rr] = (a0 + a1) + (a2 + a3);
            }
        }
        if (tid == 0) GDN_TRACE_AT(3);
    } else {
        // ---- Qt = e^G Q over the Q tile in place -> bulk store; Aqk rows staged in the same
        //      area -> bulk store, then the V tile is loaded into it; Kt = e^(G_last - G) K over
        //      the K tile in place -> bulk store, then the K tile is loaded again; finally
        //      V~ = diag(beta) V and K~ = diag(beta e^G) K in place, the B operands of U = T V~
        //      and W = T K~
        const float Gr = sG[r];
        const float fq = __expf(fminf(Gr, 0.0f));
#pragma unroll 4
        for (int c = 0; c < 16; ++c) {
            uint4 *pq = reinterpret_cast<uint4 *>(sm + OFF_QV + tile_off(128, r, c));
            const uint4 uq = *pq;
            const uint32_t wq[4] = {uq.x, uq.y, uq.z, uq.w};
            uint32_t oq[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 xq = unpack_half2(wq[e]);
                oq[e] = pack_half2(xq.x * fq, xq.y * fq);
            }
            *pq = make_uint4(oq[0], oq[1], oq[2], oq[3]);
        }
        fence_proxy_async();
        group_sync(2);
        if (tid == 128) {
            tma_store_2d(&tmQt, sm + OFF_QV, 0, y0);
            tma_store_2d(&tmQt, sm + OFF_QV + 16384, 64, y0);
            bulk_commit();
            bulk_wait_read_all();
        }
        group_sync(2);
        const int w = warp & 3;  // rows 32w .. 32w+31: same split of the decay as the L rows
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
            float a[32];
            if (c > w) {
#pragma unroll
                for (int i = 0; i < 32; ++i) a[i] = 0.0f;
            } else {
                tmem_ld32(tmem + lane_base + TM_QK + c * 32, a);
                if (c < w) {
                    const float fr = __expf(fminf(Gr - sG[c * 32 + 31], 0.0f));
#pragma unroll
                    for (int i = 0; i < 32; ++i) a[i] *= fr * sEc[c * 32 + i];
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int j = c * 32 + i;
                        a[i] = (j <= r) ? __expf(fminf(Gr - sG[j], 0.0f)) * a[i] : 0.0f;
                    }
                }
            }
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) put8(sm + OFF_QV, 128, r, c * 4 + q4, &a[q4 * 8]);
        }
        fence_proxy_async();
        group_sync(2);
        if (tid == 128) {
            tma_store_2d(&tmAqk, sm + OFF_QV, 0, y0);
            tma_store_2d(&tmAqk, sm + OFF_QV + 16384, 64, y0);
            bulk_commit();
            bulk_wait_read_all();
            mbar_arrive_expect_tx(bar_v, 32768u);
            tma_load_2d(sm + OFF_QV, &tmV, bar_v, 0, y0);
            tma_load_2d(sm + OFF_QV + 16384, &tmV, bar_v, 64, y0);
        }
        // Kt (the K tile's last use as plain K was the A_kk product, complete before this branch)
        const float fk = __expf(fminf(sG[kBlk - 1] - Gr, 0.0f));
#pragma unroll 4
        for (int c = 0; c < 16; ++c) {
            uint4 *pk = reinterpret_cast<uint4 *>(sm + OFF_K + tile_off(128, r, c));
            const uint4 uk = *pk;
            const uint32_t wk[4] = {uk.x, uk.y, uk.z, uk.w};
            uint32_t o4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 xk = unpack_half2(wk[e]);
                o4[e] = pack_half2(xk.x * fk, xk.y * fk);
            }
            *pk = make_uint4(o4[0], o4[1], o4[2], o4[3]);
        }
        fence_proxy_async();
        group_sync(2);
        if (tid == 128) {
            tma_store_2d(&tmKt, sm + OFF_K, 0, y0);
            tma_store_2d(&tmKt, sm + OFF_K + 16384, 64, y0);
            bulk_commit();
            bulk_wait_read_all();
            mbar_arrive_expect_tx(bar_kr, 32768u);
            tma_load_2d(sm + OFF_K, &tmK, bar_kr, 0, y0);
            tma_load_2d(sm + OFF_K + 16384, &tmK, bar_kr, 64, y0);
        }
        // V~ and K~, row r each
        const float sv = sBeta[r], sk = sBeta[r] * fq;
        if (mbar_wait(bar_v, 0, ab, p.status, p.wait_limit_ns)) {
#pragma unroll 4
            for (int c = 0; c < 16; ++c) {
                uint4 *pv = reinterpret_cast<uint4 *>(sm + OFF_QV + tile_off(128, r, c));
                const uint4 uv = *pv;
                const uint32_t wv[4] = {uv.x, uv.y, uv.z, uv.w};
                uint32_t o4[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 xv = unpack_half2(wv[e]);
                    o4[e] = pack_half2(xv.x * sv, xv.y * sv);
                }
                *pv = make_uint4(o4[0], o4[1], o4[2], o4[3]);
            }
        }
        if (mbar_wait(bar_kr, 0, ab, p.status, p.wait_limit_ns)) {
#pragma unroll 4
            for (int c = 0; c < 16; ++c) {
                uint4 *pk = reinterpret_cast<uint4 *>(sm + OFF_K + tile_off(128, r, c));
                const uint4 uk = *pk;
                const uint32_t wk[4] = {uk.x, uk.y, uk.z, uk.w};
                uint32_t o4[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 xk = unpack_half2(wk[e]);
                    o4[e] = pack_half2(xk.x * sk, xk.y * sk);
                }
                *pk = make_uint4(o4[0], o4[1], o4[2], o4[3]);
            }
        }
        fence_proxy_async();
    }
    tc_fence_before();
    __syncthreads();
    if (tid == 0) GDN_TRACE_AT(4);

    // ---- merge: Y = [. ; L_21] T_1 (rows 64..127 are P = L_21 T_1), then T_21^T = -P^T T_2^T
    if (groupL && r < 64) {  // T_1^T as the K-major B operand: row i = column i of T_1
#pragma unroll
        for (int c = 0; c < 8; ++c) put8(sm + OFF_T1, 64, r, c, &col[c * 8]);
    }
    fence_proxy_async();
    __syncthreads();
    if (tid == 0) {
        tc_fence_after();
        const uint32_t idesc = idesc_f16_f32(128, 64, false, false);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            umma_f16(tmem + TM_Y, sdesc_sw128(sbase + OFF_LHA + kk * 32, 16, 1024),
                     sdesc_sw128(sbase + OFF_T1 + kk * 32, 16, 1024), idesc, kk > 0);
        umma_commit(bar_mma);
    }
    if (groupL && r >= 64) {  // T_2^T as the MN-major B operand: row j' = column j' of T_2
#pragma unroll
        for (int c = 0; c < 8; ++c) put8(sm + OFF_T2T, 64, r - 64, c, &col[c * 8]);
    }
    mbar_wait(bar_mma, mma_phase, ab, p.status, p.wait_limit_ns);
    mma_phase ^= 1;
    __syncthreads();
    if (ab->flag) goto teardown;
    tc_fence_after();
    if (groupL && r >= 64) {  // [P | 0] as the MN-major A operand: row j' holds P[j'][0..63] at M = 0..63
        const int jp = r - 64;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            float a[32];
            tmem_ld32(tmem + lane_base + TM_Y + c * 32, a);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) put8(sm + OFF_PA, 64, jp, c * 4 + q4, &a[q4 * 8]);
        }
#pragma unroll
        for (int c = 8; c < 16; ++c)
            *reinterpret_cast<uint4 *>(sm + OFF_PA + tile_off(64, jp, c)) = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
        // D2[j][r'] = sum_j' P[j'][j] T_2[r'][j'] = (T_2 P)[r'][j] = -T_21[r'][j]
        tc_fence_after();
        const uint32_t idesc = idesc_f16_f32(128, 64, true, true);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            umma_f16(tmem + TM_D2, sdesc_sw128(sbase + OFF_PA + kk * 2048, 8192, 1024),
                     sdesc_sw128(sbase + OFF_T2T + kk * 2048, 8192, 1024), idesc, kk > 0);
        umma_commit(bar_mma);
    }
    mbar_wait(bar_mma, mma_phase, ab, p.status, p.wait_limit_ns);
    mma_phase ^= 1;
    __syncthreads();
    if (ab->flag) goto teardown;
    tc_fence_after();
    if (tid == 0) GDN_TRACE_AT(5);

    // ---- U = T V~ and W = T K~, one commit: A = T^T (MN-major, shared), B = the V~ / K~ tiles
    //      (MN-major)
    if (groupL) build_tT(sm + OFF_A, r, col, 1.0f, tmem + lane_base + TM_D2);
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    if (ab->flag) goto teardown;
    if (tid == 0) GDN_TRACE_AT(6);
    if (tid == 0) {
        tc_fence_after();
        const uint32_t idesc = idesc_f16_f32(128, 128, true, true);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
            umma_f16(tmem + TM_U, sdesc_sw128(sbase + OFF_A + kk * 2048, 16384, 1024),
                     sdesc_sw128(sbase + OFF_QV + kk * 2048, 16384, 1024), idesc, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
            umma_f16(tmem + TM_W, sdesc_sw128(sbase + OFF_A + kk * 2048, 16384, 1024),
                     sdesc_sw128(sbase + OFF_K + kk * 2048, 16384, 1024), idesc, kk > 0);
        umma_commit(bar_mma);
    }
    mbar_wait(bar_mma, mma_phase, ab, p.status, p.wait_limit_ns);
    mma_phase ^= 1;
    __syncthreads();
    if (ab->flag) goto teardown;
    tc_fence_after();
    if (tid == 0) GDN_TRACE_AT(7);
    // ---- W rows (group L) into the A area, U rows (group Q) into the V~ area; bulk stores
    {
        uint8_t *dst = sm + (groupL ? OFF_A : OFF_QV);
        const uint32_t tcol = groupL ? TM_W : TM_U;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
            float a[32];
            tmem_ld32(tmem + lane_base + tcol + c * 32, a);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) put8(dst, 128, r, c * 4 + q4, &a[q4 * 8]);
        }
    }
    fence_proxy_async();
    __syncthreads();
    if (tid == 0) {
        tma_store_2d(&tmW, sm + OFF_A, 0, y0);
        tma_store_2d(&tmW, sm + OFF_A + 16384, 64, y0);
        bulk_commit();
    }
    if (tid == 128) {
        tma_store_2d(&tmU, sm + OFF_QV, 0, y0);
        tma_store_2d(&tmU, sm + OFF_QV + 16384, 64, y0);
        bulk_commit();
    }
    if (tid == 0) GDN_TRACE_AT(8);

teardown:
    if (tid == 0 || tid == 128) bulk_wait_all();  // every bulk store issued by this CTA has completed
    if (tid == 0) GDN_TRACE_AT(9);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

}  // namespace

cudaError_t launch_chunk(const ChunkParams &p, const CUtensorMap &tmK, const CUtensorMap &tmV,
                         const CUtensorMap &tmQ, const CUtensorMap &tmW, const CUtensorMap &tmU,
                         const CUtensorMap &tmQt, const CUtensorMap &tmKt, const CUtensorMap &tmAqk,
                         cudaStream_t s) {
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(gdn_chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(SMEM_BYTES));
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    dim3 grid(p.NB, p.BH);
    gdn_chunk_kernel<<<grid, 256, SMEM_BYTES, s>>>(p, tmK, tmV, tmQ, tmW, tmU, tmQt, tmKt, tmAqk);
    return cudaGetLastError();
}

}  // namespace gdn

GDN_TRACE_EXPORT(chunk)
