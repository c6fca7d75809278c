// gdn_scan.cu -- K3 of the GDN forward: the inter-block state scan of the
// gated delta rule (reference [57] on the VMonarch page) and the block
// outputs, on 5th-generation tensor cores.  One CTA carries the fp32 state
// S (d_v x d_k = 128 x 128) of one (b, h) through its 128-token blocks:
//
//   X     = W S^T                     (tcgen05, TMEM)
//   Delta = U - X                     (consumer warps, fp32 -> fp16 operand)
//   S^T  <- e^(G_last) S^T + Kt^T Delta   (tcgen05 for Kt^T Delta; the fp32
//                                        state lives in the consumer threads'
//                                        registers, one d_k row per thread)
//   O     = Qt S^T + Aqk Delta        (tcgen05, accumulated in TMEM)
//
// with Kt = diag(e^(G_last - G)) K, Qt = diag(e^G) Q and Aqk the decay-masked
// Q K^T from the chunk kernel.  Warp 4 is the producer: one lane issues the
// TMA loads of the next block as soon as each tile's last reader has
// finished, and issues every MMA.  Warps 0-3 are the consumers: thread r owns
// TMEM lane r.  All hand-offs are mbarriers with bounded waits, so a lost
// arrival ends the kernel with a timeout status instead of a hang.
#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr uint32_t OFF_W = 0;
constexpr uint32_t OFF_QT = 32768;
constexpr uint32_t OFF_KT = 65536;
constexpr uint32_t OFF_AQK = 98304;
constexpr uint32_t OFF_U = 131072;
constexpr uint32_t OFF_S = 163840;   // S^T as fp16 MN-major B operand (rows d_k, cols d_v)
constexpr uint32_t OFF_D = 196608;   // Delta as fp16 MN-major B operand (rows token, cols d_v)
constexpr uint32_t OFF_BAR = 229376;
constexpr int NBAR = 11;
constexpr uint32_t SMEM_USED = OFF_BAR + NBAR * 8 + 16;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;

enum { B_FULL_WQ = 0, B_FULL_U, B_FULL_KA, B_MMA_X, B_MMA_P, B_MMA_O, B_CONS_D, B_CONS_S, B_CONS_O0, B_CONS_O1, B_TEST };
constexpr uint32_t TM_X = 0, TM_P = 128, TM_O = 256;  // O double-buffered: 256 and 384

__global__ void __launch_bounds__(160, 1)
    gdn_scan_kernel(const ScanParams p, const __grid_constant__ CUtensorMap tmW,
                    const __grid_constant__ CUtensorMap tmQt, const __grid_constant__ CUtensorMap tmKt,
                    const __grid_constant__ CUtensorMap tmAqk, const __grid_constant__ CUtensorMap tmU) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + NBAR);
    AbortState *ab = reinterpret_cast<AbortState *>(tmem_slot + 1);

    const int h = blockIdx.x, b = blockIdx.y;
    const int bh = b * p.H + h;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int NB = p.NB;
    const uint64_t lim = p.wait_limit_ns;

    if (tid == 0) {
        for (int i = 0; i < NBAR; ++i) mbar_init(&bars[i], (i >= B_CONS_D && i <= B_CONS_O1) ? 4 : 1);
        ab->flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 4) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            bool ok = true;
            if (p.test_wait_timeout) ok = mbar_wait(&bars[B_TEST], 0, ab, p.status, 50ull * 1000 * 1000);
            const int rowbase = bh * p.Tp;
            auto load_wq = [&](int c) {
                mbar_arrive_expect_tx(&bars[B_FULL_WQ], 65536);
                const int y = rowbase + c * kBlk;
                tma_load_2d(sm + OFF_W, &tmW, &bars[B_FULL_WQ], 0, y);
                tma_load_2d(sm + OFF_W + 16384, &tmW, &bars[B_FULL_WQ], 64, y);
                tma_load_2d(sm + OFF_QT, &tmQt, &bars[B_FULL_WQ], 0, y);
                tma_load_2d(sm + OFF_QT + 16384, &tmQt, &bars[B_FULL_WQ], 64, y);
            };
            auto load_u = [&](int c) {
                mbar_arrive_expect_tx(&bars[B_FULL_U], 32768);
                const int y = rowbase + c * kBlk;
                tma_load_2d(sm + OFF_U, &tmU, &bars[B_FULL_U], 0, y);
                tma_load_2d(sm + OFF_U + 16384, &tmU, &bars[B_FULL_U], 64, y);
            };
            auto load_ka = [&](int c) {
                mbar_arrive_expect_tx(&bars[B_FULL_KA], 65536);
                const int y = rowbase + c * kBlk;
                tma_load_2d(sm + OFF_KT, &tmKt, &bars[B_FULL_KA], 0, y);
                tma_load_2d(sm + OFF_KT + 16384, &tmKt, &bars[B_FULL_KA], 64, y);
                tma_load_2d(sm + OFF_AQK, &tmAqk, &bars[B_FULL_KA], 0, y);
                tma_load_2d(sm + OFF_AQK + 16384, &tmAqk, &bars[B_FULL_KA], 64, y);
            };
            if (ok) {
                load_wq(0);
                load_u(0);
                load_ka(0);
            }
            const uint32_t id_kmn = idesc_f16_f32(128, 128, false, true);
            const uint32_t id_mnmn = idesc_f16_f32(128, 128, true, true);
            for (int c = 0; ok && c < NB; ++c) {
                const uint32_t ph = c & 1;
                const uint32_t tO = tmem + TM_O + (c & 1) * 128;
                ok = mbar_wait(&bars[B_FULL_WQ], ph, ab, p.status, lim) &&
                     mbar_wait(&bars[B_CONS_S], ph, ab, p.status, lim) &&
                     (c < 2 || mbar_wait(&bars[B_CONS_O0 + (c & 1)], ((c >> 1) - 1) & 1, ab, p.status, lim));
                if (!ok) break;
                tc_fence_after();
                // X = W S^T ; O = Qt S^T   (A K-major, B = S^T MN-major)
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t aoff = (kk >> 2) * 16384 + (kk & 3) * 32;
                    const uint64_t bd = sdesc_sw128(sbase + OFF_S + kk * 2048, 16384, 1024);
                    umma_f16(tmem + TM_X, sdesc_sw128(sbase + OFF_W + aoff, 16, 1024), bd, id_kmn, kk > 0);
                    umma_f16(tO, sdesc_sw128(sbase + OFF_QT + aoff, 16, 1024), bd, id_kmn, kk > 0);
                }
                umma_commit(&bars[B_MMA_X]);
                ok = mbar_wait(&bars[B_MMA_X], ph, ab, p.status, lim);
                if (!ok) break;
                if (c + 1 < NB) load_wq(c + 1);
                ok = mbar_wait(&bars[B_FULL_KA], ph, ab, p.status, lim) &&
                     mbar_wait(&bars[B_CONS_D], ph, ab, p.status, lim);
                if (!ok) break;
                if (c + 1 < NB) load_u(c + 1);
                tc_fence_after();
                // P = Kt^T Delta  (A = Kt read MN-major: M = d_k, K = token; B = Delta MN-major)
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    umma_f16(tmem + TM_P, sdesc_sw128(sbase + OFF_KT + kk * 2048, 16384, 1024),
                             sdesc_sw128(sbase + OFF_D + kk * 2048, 16384, 1024), id_mnmn, kk > 0);
                umma_commit(&bars[B_MMA_P]);
                // O += Aqk Delta  (A K-major: M = token r, K = token i)
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t aoff = (kk >> 2) * 16384 + (kk & 3) * 32;
                    umma_f16(tO, sdesc_sw128(sbase + OFF_AQK + aoff, 16, 1024),
                             sdesc_sw128(sbase + OFF_D + kk * 2048, 16384, 1024), id_kmn, 1);
                }
                umma_commit(&bars[B_MMA_O]);
                ok = mbar_wait(&bars[B_MMA_O], ph, ab, p.status, lim);
                if (!ok) break;
                if (c + 1 < NB) load_ka(c + 1);
            }
        }
    } else {
        // ----------------------------------------------------------- consumers
        const int r = tid;  // TMEM lane: token row (X, O) or d_k row (P)
        const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
        float S[128];  // row r of S^T (= column r of S), fp32
#pragma unroll
        for (int i = 0; i < 128; ++i) S[i] = 0.0f;
#pragma unroll
        for (int c16 = 0; c16 < 16; ++c16)
            *reinterpret_cast<uint4 *>(sm + OFF_S + tile_off(128, r, c16)) = make_uint4(0, 0, 0, 0);
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[B_CONS_S]);

        const float *Gbh = p.G + static_cast<size_t>(bh) * p.Tp;
        for (int c = 0; c < NB; ++c) {
            const uint32_t ph = c & 1;
            const float gC = __expf(fminf(Gbh[c * kBlk + kBlk - 1], 0.0f));
            // every wait below is made warp-uniform before the .sync.aligned TMEM loads
            if (!__all_sync(0xffffffffu, mbar_wait(&bars[B_MMA_X], ph, ab, p.status, lim) &&
                                             mbar_wait(&bars[B_FULL_U], ph, ab, p.status, lim)))
                break;
            tc_fence_after();
            // Delta = U - X, row r
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                float x[32];
                tmem_ld32(tmem + lane_base + TM_X + ch * 32, x);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint32_t off = tile_off(128, r, ch * 4 + q);
                    const uint4 uu = *reinterpret_cast<const uint4 *>(sm + OFF_U + off);
                    const uint32_t w[4] = {uu.x, uu.y, uu.z, uu.w};
                    uint32_t o[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 u2 = unpack_half2(w[e]);
                        o[e] = pack_half2(u2.x - x[q * 8 + 2 * e], u2.y - x[q * 8 + 2 * e + 1]);
                    }
                    *reinterpret_cast<uint4 *>(sm + OFF_D + off) = make_uint4(o[0], o[1], o[2], o[3]);
                }
            }
            fence_proxy_async();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_CONS_D]);

            // S^T row r <- gC * S^T row r + P row r
            if (!__all_sync(0xffffffffu, mbar_wait(&bars[B_MMA_P], ph, ab, p.status, lim))) break;
            tc_fence_after();
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                float pv[32];
                tmem_ld32(tmem + lane_base + TM_P + ch * 32, pv);
#pragma unroll
                for (int i = 0; i < 32; ++i) S[ch * 32 + i] = fmaf(gC, S[ch * 32 + i], pv[i]);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int e0 = ch * 32 + q * 8;
                    uint4 u;
                    u.x = pack_half2(S[e0 + 0], S[e0 + 1]);
                    u.y = pack_half2(S[e0 + 2], S[e0 + 3]);
                    u.z = pack_half2(S[e0 + 4], S[e0 + 5]);
                    u.w = pack_half2(S[e0 + 6], S[e0 + 7]);
                    *reinterpret_cast<uint4 *>(sm + OFF_S + tile_off(128, r, ch * 4 + q)) = u;
                }
            }
            fence_proxy_async();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_CONS_S]);

            // block output rows
            if (!__all_sync(0xffffffffu, mbar_wait(&bars[B_MMA_O], ph, ab, p.status, lim))) break;
            tc_fence_after();
            const int t = c * kBlk + r;
            float *orow = p.o + ((static_cast<size_t>(b) * p.T + t) * p.H + h) * kD;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                float ov[32];
                tmem_ld32(tmem + lane_base + TM_O + (c & 1) * 128 + ch * 32, ov);
                if (t < p.T) {
#pragma unroll
                    for (int i = 0; i < 32; i += 4)
                        *reinterpret_cast<float4 *>(orow + ch * 32 + i) = make_float4(ov[i], ov[i + 1], ov[i + 2], ov[i + 3]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_CONS_O0 + (c & 1)]);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace

cudaError_t launch_scan(const ScanParams &p, const CUtensorMap &tmW, const CUtensorMap &tmQt,
                        const CUtensorMap &tmKt, const CUtensorMap &tmAqk, const CUtensorMap &tmU,
                        cudaStream_t s) {
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(gdn_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(SMEM_BYTES));
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    dim3 grid(p.H, p.B);
    gdn_scan_kernel<<<grid, 160, SMEM_BYTES, s>>>(p, tmW, tmQt, tmKt, tmAqk, tmU);
    return cudaGetLastError();
}

}  // namespace gdn
