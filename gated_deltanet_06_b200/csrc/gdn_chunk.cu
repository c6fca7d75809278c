// gdn_chunk.cu -- K2 of the GDN forward: the intra-block UT (WY) transform of
// the gated delta rule (reference [57] on the VMonarch page) on 5th-generation
// tensor cores.  One CTA handles one 128-token block of one (b, h):
//
//   A_kk = K K^T                          tcgen05, fp16 x fp16 -> fp32 in TMEM
//   L_rj = beta_r exp(G_r - G_j) A_kk,rj  for j < r (decay-masked strict tril)
//   T    = (I + L)^-1                     two 64x64 forward substitutions in
//                                         shared memory (fp32, one column per
//                                         thread) merged by
//                                         T_21 = -T_2 (L_21 T_1) on tcgen05
//   W    = T diag(beta e^G) K,  U = T diag(beta) V      tcgen05
//   Kt   = diag(e^(G_last - G)) K,  Qt = diag(e^G) Q,
//   Aqk  = [i <= r] e^(G_r - G_i) (Q K^T)_ri            tcgen05 for Q K^T
//
// and writes W, U, Kt, Qt, Aqk (fp16) for the inter-block scan.  Only
// exponentials of non-positive differences of the cumulative log decay G are
// taken.  K, V, Q tiles arrive by TMA in the 128B-swizzled layout the UMMA
// descriptors read directly; every operand the threads build is written in
// the same layout.
#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

// Shared-memory map (offsets from a 1024-byte aligned base).
constexpr uint32_t OFF_K = 0;              // 128x128 fp16 panel tile (TMA)
constexpr uint32_t OFF_V = 32768;          // 128x128 fp16 panel tile (TMA)
constexpr uint32_t OFF_Q = 65536;          // 128x128 fp16 panel tile (TMA)
constexpr uint32_t OFF_UNION = 98304;      // 80 KB, reused between phases:
constexpr uint32_t OFF_LD1 = OFF_UNION + 0;       //   fp32 64x64, L diagonal block 1
constexpr uint32_t OFF_LD2 = OFF_UNION + 16384;   //   fp32 64x64, L diagonal block 2
constexpr uint32_t OFF_LH = OFF_UNION + 32768;    //   fp16 128 rows x 64 (L[:, 0:64]), K-major A
constexpr uint32_t OFF_T1 = OFF_UNION + 49152;    //   fp16 64 x 64 (T_1^T), K-major B
constexpr uint32_t OFF_T2 = OFF_UNION + 57344;    //   fp16 64 rows x 128 ([0; T_2]), MN-major A
constexpr uint32_t OFF_P = OFF_UNION + 73728;     //   fp16 64 x 64 (L_21 T_1), MN-major B
constexpr uint32_t OFF_AQK = OFF_UNION + 49152;   //   fp16 128x128 Aqk staging for the bulk store
                                                  //   (done reading before T_1/T_2/P are written)
constexpr uint32_t OFF_A1 = OFF_UNION + 0;        //   fp16 128x128 T diag(beta e^G), K-major A
constexpr uint32_t OFF_A2 = OFF_UNION + 32768;    //   fp16 128x128 T diag(beta), K-major A
constexpr uint32_t OFF_G = OFF_UNION + 81920;     // fp32 [128]
constexpr uint32_t OFF_BETA = OFF_G + 512;        // fp32 [128]
constexpr uint32_t OFF_BAR = OFF_BETA + 512;      // 2 mbarriers, tmem slot, abort flag
constexpr uint32_t SMEM_USED = OFF_BAR + 32;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // + alignment slack

constexpr uint32_t TM_AKK = 0, TM_QK = 128, TM_Y = 256, TM_T2P = 320, TM_W = 0, TM_U = 128;

__global__ void __launch_bounds__(128, 1)
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
    uint64_t *bar_load = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    uint64_t *bar_mma = bar_load + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_load + 2);
    AbortState *ab = reinterpret_cast<AbortState *>(tmem_slot + 1);

    const int blk = blockIdx.x, bh = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int r = tid;  // TMEM lane / row owned by this thread
    const size_t row0 = static_cast<size_t>(bh) * p.Tp + static_cast<size_t>(blk) * kBlk;

    if (tid == 0) {
        mbar_init(bar_load, 1);
        mbar_init(bar_mma, 1);
        ab->flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    sG[tid] = p.G[row0 + tid];
    sBeta[tid] = p.beta[row0 + tid];
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    uint32_t mma_phase = 0;

    if (tid == 0) {
        mbar_arrive_expect_tx(bar_load, 3u * 32768u);
        const int y = static_cast<int>(row0);
        tma_load_2d(sm + OFF_K, &tmK, bar_load, 0, y);
        tma_load_2d(sm + OFF_K + 16384, &tmK, bar_load, 64, y);
        tma_load_2d(sm + OFF_V, &tmV, bar_load, 0, y);
        tma_load_2d(sm + OFF_V + 16384, &tmV, bar_load, 64, y);
        tma_load_2d(sm + OFF_Q, &tmQ, bar_load, 0, y);
        tma_load_2d(sm + OFF_Q + 16384, &tmQ, bar_load, 64, y);
    }
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
            umma_f16(tmem + TM_QK, sdesc_sw128(sbase + OFF_Q + koff, 16, 1024), dk, idesc, kk > 0);
        }
        umma_commit(bar_mma);
    }
    mbar_wait(bar_mma, mma_phase, ab, p.status, p.wait_limit_ns);
    mma_phase ^= 1;
    __syncthreads();
    if (ab->flag) goto teardown;
    tc_fence_after();

    {
        const float Gr = sG[r], br = sBeta[r];
        float *Ld1 = reinterpret_cast<float *>(sm + OFF_LD1);
        float *Ld2 = reinterpret_cast<float *>(sm + OFF_LD2);
        // L row r: fp32 diagonal blocks for the solves, fp16 left half for L_21 T_1
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
            float a[32];
            tmem_ld32(tmem + lane_base + TM_AKK + c * 32, a);
            float l[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const int j = c * 32 + i;
                l[i] = (j < r) ? br * __expf(fminf(Gr - sG[j], 0.0f)) * a[i] : 0.0f;
            }
            if (c < 2) {
                if (r < 64) {
#pragma unroll
                    for (int i = 0; i < 32; i += 4)
                        *reinterpret_cast<float4 *>(Ld1 + r * 64 + c * 32 + i) =
                            make_float4(l[i], l[i + 1], l[i + 2], l[i + 3]);
                }
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    uint4 u;
                    u.x = pack_half2(l[q4 * 8 + 0], l[q4 * 8 + 1]);
                    u.y = pack_half2(l[q4 * 8 + 2], l[q4 * 8 + 3]);
                    u.z = pack_half2(l[q4 * 8 + 4], l[q4 * 8 + 5]);
                    u.w = pack_half2(l[q4 * 8 + 6], l[q4 * 8 + 7]);
                    *reinterpret_cast<uint4 *>(sm + OFF_LH + tile_off(128, r, c * 4 + q4)) = u;
                }
            } else if (r >= 64) {
#pragma unroll
                for (int i = 0; i < 32; i += 4)
                    *reinterpret_cast<float4 *>(Ld2 + (r - 64) * 64 + (c - 2) * 32 + i) =
                        make_float4(l[i], l[i + 1], l[i + 2], l[i + 3]);
            }
        }
        // Aqk row r (staged for a bulk store); Qt = e^G Q written over the Q tile in place
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
            float a[32];
            tmem_ld32(tmem + lane_base + TM_QK + c * 32, a);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const int j = c * 32 + i;
                a[i] = (j <= r) ? __expf(fminf(Gr - sG[j], 0.0f)) * a[i] : 0.0f;
            }
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                uint4 u;
                u.x = pack_half2(a[q4 * 8 + 0], a[q4 * 8 + 1]);
                u.y = pack_half2(a[q4 * 8 + 2], a[q4 * 8 + 3]);
                u.z = pack_half2(a[q4 * 8 + 4], a[q4 * 8 + 5]);
                u.w = pack_half2(a[q4 * 8 + 6], a[q4 * 8 + 7]);
                *reinterpret_cast<uint4 *>(sm + OFF_AQK + tile_off(128, r, c * 4 + q4)) = u;
            }
        }
        const float fq = __expf(fminf(Gr, 0.0f));
#pragma unroll 4
        for (int c = 0; c < 16; ++c) {
            uint4 *pq = reinterpret_cast<uint4 *>(sm + OFF_Q + tile_off(128, r, c));
            const uint4 uq = *pq;
            const uint32_t wq[4] = {uq.x, uq.y, uq.z, uq.w};
            uint32_t oq[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 xq = unpack_half2(wq[i]);
                oq[i] = pack_half2(xq.x * fq, xq.y * fq);
            }
            *pq = make_uint4(oq[0], oq[1], oq[2], oq[3]);
        }
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
        const int y = static_cast<int>(row0);
        tma_store_2d(&tmAqk, sm + OFF_AQK, 0, y);
        tma_store_2d(&tmAqk, sm + OFF_AQK + 16384, 64, y);
        tma_store_2d(&tmQt, sm + OFF_Q, 0, y);
        tma_store_2d(&tmQt, sm + OFF_Q + 16384, 64, y);
        bulk_commit();
    }

    if (tid == 0) GDN_TRACE_AT(2);
    // ---- two 64x64 unit lower-triangular inverses, one column per thread
    float col[64];
    {
        const int i = r & 63;
        const float *Ld = reinterpret_cast<const float *>(sm + (r < 64 ? OFF_LD1 : OFF_LD2));
        // four independent partial sums per row keep the FMA pipe busy
#pragma unroll
        for (int rr = 0; rr < 64; ++rr) {
            float a0 = (rr == i) ? 1.0f : 0.0f, a1 = 0.0f, a2 = 0.0f, a3 = 0.0f;
#pragma unroll
            for (int j4 = 0; j4 < rr; j4 += 4) {
                const float4 l = *reinterpret_cast<const float4 *>(Ld + rr * 64 + j4);
                a0 = fmaf(-l.x, col[j4], a0);
                if (j4 + 1 < rr) a1 = fmaf(-l.y, col[j4 + 1], a1);
                if (j4 + 2 < rr) a2 = fmaf(-l.z, col[j4 + 2], a2);
                if (j4 + 3 < rr) a3 = fmaf(-l.w, col[j4 + 3], a3);
            }
            col[rr] = (a0 + a1) + (a2 + a3);
        }
    }
    if (tid == 0) GDN_TRACE_AT(3);
    // T_1, T_2, P below overwrite the Aqk staging area: the bulk store must have read it
    if (tid == 0) bulk_wait_read_all();
    if (tid == 0) GDN_TRACE_AT(4);
    __syncthreads();
    // T_1^T as the K-major B operand (row i = column i of T_1)
    if (r < 64) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            uint4 u;
            u.x = pack_half2(col[c * 8 + 0], col[c * 8 + 1]);
            u.y = pack_half2(col[c * 8 + 2], col[c * 8 + 3]);
            u.z = pack_half2(col[c * 8 + 4], col[c * 8 + 5]);
            u.w = pack_half2(col[c * 8 + 6], col[c * 8 + 7]);
            *reinterpret_cast<uint4 *>(sm + OFF_T1 + tile_off(64, r, c)) = u;
        }
    }
    fence_proxy_async();
    __syncthreads();
    // ---- Y = L[:, 0:64] T_1   (rows 64..127 of Y are L_21 T_1)
    if (tid == 0) {
        tc_fence_after();
        const uint32_t idesc = idesc_f16_f32(128, 64, false, false);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            umma_f16(tmem + TM_Y, sdesc_sw128(sbase + OFF_LH + kk * 32, 16, 1024),
                     sdesc_sw128(sbase + OFF_T1 + kk * 32, 16, 1024), idesc, kk > 0);
        umma_commit(bar_mma);
    }
    // [0; T_2] as the MN-major A operand: row j' holds column j' of T_2 at M = 64..127
    if (r >= 64) {
        const int jp = r - 64;
#pragma unroll
        for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4 *>(sm + OFF_T2 + tile_off(64, jp, c)) = make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            uint4 u;
            u.x = pack_half2(col[c * 8 + 0], col[c * 8 + 1]);
            u.y = pack_half2(col[c * 8 + 2], col[c * 8 + 3]);
            u.z = pack_half2(col[c * 8 + 4], col[c * 8 + 5]);
            u.w = pack_half2(col[c * 8 + 6], col[c * 8 + 7]);
            *reinterpret_cast<uint4 *>(sm + OFF_T2 + tile_off(64, jp, 8 + c)) = u;
        }
    }
    mbar_wait(bar_mma, mma_phase, ab, p.status, p.wait_limit_ns);
    mma_phase ^= 1;
    __syncthreads();
    if (ab->flag) goto teardown;
    tc_fence_after();
    // P = L_21 T_1 (rows 64..127 of Y) as the MN-major B operand
    if (warp >= 2) {
        const int jp = r - 64;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            float a[32];
            tmem_ld32(tmem + lane_base + TM_Y + c * 32, a);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                uint4 u;
                u.x = pack_half2(a[q4 * 8 + 0], a[q4 * 8 + 1]);
                u.y = pack_half2(a[q4 * 8 + 2], a[q4 * 8 + 3]);
                u.z = pack_half2(a[q4 * 8 + 4], a[q4 * 8 + 5]);
                u.w = pack_half2(a[q4 * 8 + 6], a[q4 * 8 + 7]);
                *reinterpret_cast<uint4 *>(sm + OFF_P + tile_off(64, jp, c * 4 + q4)) = u;
            }
        }
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    // ---- T_2 P  (rows 64..127); T_21 = -T_2 P
    if (tid == 0) {
        tc_fence_after();
        const uint32_t idesc = idesc_f16_f32(128, 64, true, true);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            umma_f16(tmem + TM_T2P, sdesc_sw128(sbase + OFF_T2 + kk * 2048, 8192, 1024),
                     sdesc_sw128(sbase + OFF_P + kk * 2048, 8192, 1024), idesc, kk > 0);
        umma_commit(bar_mma);
    }
    mbar_wait(bar_mma, mma_phase, ab, p.status, p.wait_limit_ns);
    mma_phase ^= 1;
    __syncthreads();
    if (ab->flag) goto teardown;
    tc_fence_after();

    if (tid == 0) GDN_TRACE_AT(5);
    // ---- A1 = T diag(beta e^G), A2 = T diag(beta): K-major A operands (row r, column j)
    {
        uint8_t *A1 = sm + OFF_A1;
        uint8_t *A2 = sm + OFF_A2;
        if (r < 64) {
            // columns 64..127 of rows 0..63 are zero
#pragma unroll
            for (int c = 8; c < 16; ++c) {
                *reinterpret_cast<uint4 *>(A1 + tile_off(128, r, c)) = make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4 *>(A2 + tile_off(128, r, c)) = make_uint4(0, 0, 0, 0);
            }
        } else {
            // row r of T_21 = -(T_2 P) row r, scaled by column
            const int rr = r;
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                float a[32];
                tmem_ld32(tmem + lane_base + TM_T2P + c * 32, a);
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    float v1[8], v2[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int j = c * 32 + q4 * 8 + e;
                        const float t = -a[q4 * 8 + e];
                        v2[e] = t * sBeta[j];
                        v1[e] = v2[e] * __expf(fminf(sG[j], 0.0f));
                    }
                    uint4 u1, u2;
                    u1.x = pack_half2(v1[0], v1[1]); u1.y = pack_half2(v1[2], v1[3]);
                    u1.z = pack_half2(v1[4], v1[5]); u1.w = pack_half2(v1[6], v1[7]);
                    u2.x = pack_half2(v2[0], v2[1]); u2.y = pack_half2(v2[2], v2[3]);
                    u2.z = pack_half2(v2[4], v2[5]); u2.w = pack_half2(v2[6], v2[7]);
                    *reinterpret_cast<uint4 *>(A1 + tile_off(128, rr, c * 4 + q4)) = u1;
                    *reinterpret_cast<uint4 *>(A2 + tile_off(128, rr, c * 4 + q4)) = u2;
                }
            }
        }
    }
    __syncthreads();  // zero/T_21 stores precede the column scatter below only by program order per thread
    {
        // diagonal blocks: thread r holds column (r & 63) of T_1 (r < 64) or T_2 (r >= 64)
        uint8_t *A1 = sm + OFF_A1;
        uint8_t *A2 = sm + OFF_A2;
        const int j = r;  // global column index
        const float s2 = sBeta[j];
        const float s1 = s2 * __expf(fminf(sG[j], 0.0f));
        const int rbase = (r < 64) ? 0 : 64;
#pragma unroll
        for (int rr = 0; rr < 64; ++rr) {
            const uint32_t off = tile_elem_off(128, rbase + rr, j);
            *reinterpret_cast<__half *>(A1 + off) = __float2half_rn(col[rr] * s1);
            *reinterpret_cast<__half *>(A2 + off) = __float2half_rn(col[rr] * s2);
        }
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) GDN_TRACE_AT(6);
    // ---- W = A1 K, U = A2 V  (A K-major; B = the TMA tiles read MN-major: K = token, N = channel)
    if (tid == 0) {
        tc_fence_after();
        const uint32_t idesc = idesc_f16_f32(128, 128, false, true);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const uint32_t aoff = (kk >> 2) * 16384 + (kk & 3) * 32;
            umma_f16(tmem + TM_W, sdesc_sw128(sbase + OFF_A1 + aoff, 16, 1024),
                     sdesc_sw128(sbase + OFF_K + kk * 2048, 16384, 1024), idesc, kk > 0);
            umma_f16(tmem + TM_U, sdesc_sw128(sbase + OFF_A2 + aoff, 16, 1024),
                     sdesc_sw128(sbase + OFF_V + kk * 2048, 16384, 1024), idesc, kk > 0);
        }
        umma_commit(bar_mma);
    }
    mbar_wait(bar_mma, mma_phase, ab, p.status, p.wait_limit_ns);
    mma_phase ^= 1;
    __syncthreads();
    if (ab->flag) goto teardown;
    tc_fence_after();
    if (tid == 0) GDN_TRACE_AT(7);
    {
        // W -> A1 area, U -> A2 area (both free now), Kt = e^(G_last - G) K over the K tile in place
        const float fk = __expf(fminf(sG[kBlk - 1] - sG[r], 0.0f));
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
            float a[32];
            tmem_ld32(tmem + lane_base + TM_W + c * 32, a);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                uint4 u;
                u.x = pack_half2(a[q4 * 8 + 0], a[q4 * 8 + 1]);
                u.y = pack_half2(a[q4 * 8 + 2], a[q4 * 8 + 3]);
                u.z = pack_half2(a[q4 * 8 + 4], a[q4 * 8 + 5]);
                u.w = pack_half2(a[q4 * 8 + 6], a[q4 * 8 + 7]);
                *reinterpret_cast<uint4 *>(sm + OFF_A1 + tile_off(128, r, c * 4 + q4)) = u;
            }
            tmem_ld32(tmem + lane_base + TM_U + c * 32, a);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                uint4 u;
                u.x = pack_half2(a[q4 * 8 + 0], a[q4 * 8 + 1]);
                u.y = pack_half2(a[q4 * 8 + 2], a[q4 * 8 + 3]);
                u.z = pack_half2(a[q4 * 8 + 4], a[q4 * 8 + 5]);
                u.w = pack_half2(a[q4 * 8 + 6], a[q4 * 8 + 7]);
                *reinterpret_cast<uint4 *>(sm + OFF_A2 + tile_off(128, r, c * 4 + q4)) = u;
            }
        }
#pragma unroll 4
        for (int c = 0; c < 16; ++c) {
            uint4 *pk = reinterpret_cast<uint4 *>(sm + OFF_K + tile_off(128, r, c));
            const uint4 uk = *pk;
            const uint32_t wk[4] = {uk.x, uk.y, uk.z, uk.w};
            uint32_t ok4[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 xk = unpack_half2(wk[i]);
                ok4[i] = pack_half2(xk.x * fk, xk.y * fk);
            }
            *pk = make_uint4(ok4[0], ok4[1], ok4[2], ok4[3]);
        }
    }
    fence_proxy_async();
    __syncthreads();
    if (tid == 0) {
        const int y = static_cast<int>(row0);
        tma_store_2d(&tmW, sm + OFF_A1, 0, y);
        tma_store_2d(&tmW, sm + OFF_A1 + 16384, 64, y);
        tma_store_2d(&tmU, sm + OFF_A2, 0, y);
        tma_store_2d(&tmU, sm + OFF_A2 + 16384, 64, y);
        tma_store_2d(&tmKt, sm + OFF_K, 0, y);
        tma_store_2d(&tmKt, sm + OFF_K + 16384, 64, y);
        bulk_commit();
    }

    if (tid == 0) GDN_TRACE_AT(8);
teardown:
    if (tid == 0) bulk_wait_all();  // every bulk store issued by this CTA has completed
    if (tid == 0) GDN_TRACE_AT(9);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 512);
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
    gdn_chunk_kernel<<<grid, 128, SMEM_BYTES, s>>>(p, tmK, tmV, tmQ, tmW, tmU, tmQt, tmKt, tmAqk);
    return cudaGetLastError();
}

}  // namespace gdn

GDN_TRACE_EXPORT(chunk)
