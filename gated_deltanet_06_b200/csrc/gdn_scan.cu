// gdn_scan.cu -- the inter-block part of the gated delta rule (reference [57]
// on the VMonarch page) on 5th-generation tensor cores, parallel over
// segments of the sequence, and the output step.
//
// Per 128-token block c, with W, U, Kt = diag(e^(G_last - G)) K, Qt =
// diag(e^G) Q and the decay-masked Aqk from the chunk kernel, the state moves
//   Delta = U - W S^T,  S^T <- e^(G_last) S^T + Kt^T Delta,
// and the block output is O = Qt S^T + Aqk Delta.  Substituting, S_end =
// S_start P + S_loc for a run of blocks, with P = prod_c (e^(G_last) I - W^T Kt)
// and S_loc the end state from S_start = 0.  So the sequence is cut into
// segments processed in parallel:
//   pass A  (gdn_transfer_kernel): per segment, run the state and the
//           transfer together as one 256-column state [S^T | P^T] from
//           [0 | I], its two halves as independent, interleaved chains;
//           write both (fp32).  With a given initial state S_0, segment 0
//           starts from [S_0^T | I] and so ends at S_start(1) itself.
//   combine (gdn_combine_kernel): S_start(j+1)^T = P_j^T S_start(j)^T + S_loc(j)^T,
//           sequential over segments, split-precision tf32 tensor-core products
//           (close to fp32), P_j^T staged in shared memory one segment ahead.
//   pass C  (gdn_scan_out_kernel): per segment, run the state from S_start
//           (S_0 or zero for segment 0) and emit the block outputs, with the
//           output step fused into the epilogue:
//           y = o / sqrt(mean(o^2) + eps) * w * SiLU(z);
//           the last segment writes the final state when it is wanted.
// In both passes a producer warp issues the TMA loads of the next block as
// soon as each tile's last reader has finished, and all MMAs; consumer warps
// own TMEM lanes (one row each) and keep the fp32 state in TMEM.  Every
// hand-off is an mbarrier with a bounded wait, so a lost arrival ends the
// kernel with a timeout status instead of a hang.  All three kernels are
// launched behind the previous kernel with programmatic dependent launch and
// wait for it (griddepcontrol.wait) before reading its outputs.
#include <type_traits>

#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

__device__ __forceinline__ void store_f16_chunk(uint8_t *tile, int rows, int r, int chunk16, const float *v) {
    uint4 u;
    u.x = pack_half2(v[0], v[1]);
    u.y = pack_half2(v[2], v[3]);
    u.z = pack_half2(v[4], v[5]);
    u.w = pack_half2(v[6], v[7]);
    *reinterpret_cast<uint4 *>(tile + tile_off(rows, r, chunk16)) = u;
}
// as store_f16_chunk, and the same 16 bytes to global row `grow` (columns 8 chunk16 ..) when grow is set
__device__ __forceinline__ void store_f16_chunk2(uint8_t *tile, int rows, int r, int chunk16, const float *v,
                                                 __half *grow) {
    uint4 u;
    u.x = pack_half2(v[0], v[1]);
    u.y = pack_half2(v[2], v[3]);
    u.z = pack_half2(v[4], v[5]);
    u.w = pack_half2(v[6], v[7]);
    *reinterpret_cast<uint4 *>(tile + tile_off(rows, r, chunk16)) = u;
    if (grow) *reinterpret_cast<uint4 *>(grow + chunk16 * 8) = u;
}

// Warp-uniform bounded wait (every lane waits; the warp proceeds only if all did).
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t ph, volatile AbortState *ab, int *status,
                                          uint64_t lim) {
    return __all_sync(0xffffffffu, mbar_wait(bar, ph, ab, status, lim));
}

// ============================================================ pass A
namespace ta {
constexpr uint32_t OFF_W = 0, OFF_KT = 32768, OFF_U = 65536;
constexpr uint32_t OFF_Z = 98304;    // [S^T | P^T] fp16, 128 rows (d_k) x 256, MN-major B (4 panels)
constexpr uint32_t OFF_D = 163840;   // Delta fp16, 128 rows (token) x 256, MN-major B
constexpr uint32_t OFF_BAR = 229376;
constexpr int NBAR = 11;
constexpr uint32_t SMEM_BYTES = OFF_BAR + NBAR * 8 + 16 + 1024;
// The two halves of the state (S^T: columns 0-127, P^T: 128-255) evolve independently, so each
// has its own products and hand-offs (index + half): the tensor core works on one half while the
// other half's warps process theirs.
enum { FULL_W = 0, FULL_U, FULL_K, MMA_X, MMA_P = MMA_X + 2, CONS_D = MMA_P + 2, CONS_S = CONS_D + 2 };
// Per half, X and P share 128 columns (X is read out before P is written); the fp32
// state [S^T | P^T] lives in the other 256.
constexpr uint32_t TM_X = 0, TM_P = 0, TM_Z = 256;
}  // namespace ta

__global__ void __launch_bounds__(288, 1)
    gdn_transfer_kernel(const ScanParams p, const __grid_constant__ CUtensorMap tmW,
                        const __grid_constant__ CUtensorMap tmKt, const __grid_constant__ CUtensorMap tmU) {
    using namespace ta;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + NBAR);
    AbortState *ab = reinterpret_cast<AbortState *>(tmem_slot + 1);

    const int seg = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int bh = b * p.H + h;
    const int c0 = seg * p.Ls, c1 = min(c0 + p.Ls, p.NB);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint64_t lim = p.wait_limit_ns;
    // debug: the segment's blocks inside the [BH][Tp] tiles and gates, and its [S_loc^T | P^T]
    // inside Zloc
    if (!debug_in_bounds(p.debug, static_cast<size_t>(bh) * p.Tp + static_cast<size_t>(c0) * kBlk,
                         static_cast<size_t>(max(c1 - c0, 0)) * kBlk, static_cast<size_t>(p.B) * p.H * p.Tp, p.status) ||
        !debug_in_bounds(p.debug, (static_cast<size_t>(bh) * p.NS + seg) * 128 * 256, 128 * 256,
                         static_cast<size_t>(p.B) * p.H * p.NS * 128 * 256, p.status))
        return;

    if (tid == 0) {
        for (int i = 0; i < NBAR; ++i) mbar_init(&bars[i], i >= CONS_D ? 4 : 1);
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
    pdl_wait();  // the UT kernel's tiles are complete

    if (warp == 8) {
        if (lane == 0) {
            const int rowbase = bh * p.Tp;
            // phases this thread has started on each barrier it feeds (TMA loads, commits), for the
            // drain below; every phase but a barrier's last is waited on before the next starts
            int started[CONS_D] = {};
            auto load2 = [&](uint32_t off, const CUtensorMap *m, uint64_t *bar, int c) {
                mbar_arrive_expect_tx(bar, 32768);
                tma_load_2d(sm + off, m, bar, 0, rowbase + c * kBlk);
                tma_load_2d(sm + off + 16384, m, bar, 64, rowbase + c * kBlk);
                ++started[bar - bars];
            };
            load2(OFF_W, &tmW, &bars[FULL_W], c0);
            load2(OFF_U, &tmU, &bars[FULL_U], c0);
            load2(OFF_KT, &tmKt, &bars[FULL_K], c0);
            const uint32_t id_x = idesc_f16_f32(128, 128, false, true);
            const uint32_t id_p = idesc_f16_f32(128, 128, true, true);
            bool ok = true;
            for (int c = c0; ok && c < c1; ++c) {
                const uint32_t ph = (c - c0) & 1;
                if (c + 2 < c1) {  // pull the tiles of block c+2 into L2 ahead of their TMA loads
                    const int y2 = rowbase + (c + 2) * kBlk;
                    for (int hf = 0; hf < 2; ++hf) {
                        tma_prefetch_2d(&tmW, hf * 64, y2);
                        tma_prefetch_2d(&tmU, hf * 64, y2);
                        tma_prefetch_2d(&tmKt, hf * 64, y2);
                    }
                }
                ok = mbar_wait(&bars[FULL_W], ph, ab, p.status, lim);
                // X_h = W [S^T | P^T]_h  (A = W K-major, B = the half's two panels of Z, MN-major)
                for (int hf = 0; ok && hf < 2; ++hf) {
                    ok = mbar_wait(&bars[CONS_S + hf], ph, ab, p.status, lim);
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        umma_f16(tmem + TM_X + hf * 128,
                                 sdesc_sw128(sbase + OFF_W + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                                 sdesc_sw128(sbase + OFF_Z + hf * 32768 + kk * 2048, 16384, 1024), id_x, kk > 0);
                    umma_commit(&bars[MMA_X + hf]);
                    ++started[MMA_X + hf];
                }
                ok = ok && mbar_wait(&bars[MMA_X], ph, ab, p.status, lim) &&
                     mbar_wait(&bars[MMA_X + 1], ph, ab, p.status, lim);
                if (!ok) break;
                if (c + 1 < c1) load2(OFF_W, &tmW, &bars[FULL_W], c + 1);
                ok = mbar_wait(&bars[FULL_K], ph, ab, p.status, lim);
                // P_h = Kt^T Delta_h  (A = Kt MN-major: M = d_k, K = token; B = the half's panels of Delta)
                for (int hf = 0; ok && hf < 2; ++hf) {
                    ok = mbar_wait(&bars[CONS_D + hf], ph, ab, p.status, lim);
                    if (!ok) break;
                    if (hf == 0 && c + 1 < c1) load2(OFF_U, &tmU, &bars[FULL_U], c + 1);  // U's only readers are done
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        umma_f16(tmem + TM_P + hf * 128, sdesc_sw128(sbase + OFF_KT + kk * 2048, 16384, 1024),
                                 sdesc_sw128(sbase + OFF_D + hf * 32768 + kk * 2048, 16384, 1024), id_p, kk > 0);
                    umma_commit(&bars[MMA_P + hf]);
                    ++started[MMA_P + hf];
                }
                ok = ok && mbar_wait(&bars[MMA_P], ph, ab, p.status, lim) &&
                     mbar_wait(&bars[MMA_P + 1], ph, ab, p.status, lim);
                if (!ok) break;
                if (c + 1 < c1) load2(OFF_KT, &tmKt, &bars[FULL_K], c + 1);
            }
            // loads and products still in flight (after an abort) complete before shared memory and
            // TMEM go away; immediate when everything has completed
#pragma unroll 1
            for (int k = 0; k < CONS_D; ++k)
                if (started[k] > 0) mbar_wait_drain(&bars[k], (started[k] - 1) & 1, lim);
        }
    } else {
        const int q = warp & 3, half = warp >> 2;  // half 0: S^T columns, half 1: P^T columns
        const int r = q * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
        const uint32_t tz = tmem + lane_base + TM_Z + half * 128;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
            float v[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = (half == 1 && ch * 32 + e == r) ? 1.0f : 0.0f;
            if (half == 0 && seg == 0 && p.s0) {
                // a given initial state: segment 0 then ends at S_start(1) itself (S_loc(0) = s0 P_0 + S_loc)
                const float *src = p.s0 + (static_cast<size_t>(bh) * 128 + ch * 32) * 128 + r;
#pragma unroll
                for (int e = 0; e < 32; ++e) v[e] = src[static_cast<size_t>(e) * 128];
            }
            tmem_st32(tz + ch * 32, v);
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) store_f16_chunk(sm + OFF_Z, 128, r, half * 16 + ch * 4 + qq, &v[qq * 8]);
        }
        tmem_st_wait();
        fence_proxy_async();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[CONS_S + half]);
        const float *Gbh = p.G + static_cast<size_t>(bh) * p.Tp;
        bool ok = true;
        for (int c = c0; c < c1; ++c) {
            const uint32_t ph = (c - c0) & 1;
            const float gC = __expf(fminf(Gbh[c * kBlk + kBlk - 1], 0.0f));
            ok = warp_wait(&bars[MMA_X + half], ph, ab, p.status, lim) &&
                 (half == 1 || warp_wait(&bars[FULL_U], ph, ab, p.status, lim));
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                float x[32];
                tmem_ld32(tmem + lane_base + TM_X + half * 128 + ch * 32, x);
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    float dlt[8];
                    if (half == 0) {
                        const uint4 uu = *reinterpret_cast<const uint4 *>(sm + OFF_U + tile_off(128, r, ch * 4 + qq));
                        const uint32_t w4[4] = {uu.x, uu.y, uu.z, uu.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 u2 = unpack_half2(w4[e]);
                            dlt[2 * e] = u2.x - x[qq * 8 + 2 * e];
                            dlt[2 * e + 1] = u2.y - x[qq * 8 + 2 * e + 1];
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 8; ++e) dlt[e] = -x[qq * 8 + e];
                    }
                    store_f16_chunk(sm + OFF_D, 128, r, half * 16 + ch * 4 + qq, dlt);
                }
            }
            fence_proxy_async();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[CONS_D + half]);
            ok = warp_wait(&bars[MMA_P + half], ph, ab, p.status, lim);
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                float pv[32], zv[32];
                tmem_ld32(tmem + lane_base + TM_P + half * 128 + ch * 32, pv);
                tmem_ld32(tz + ch * 32, zv);
#pragma unroll
                for (int e = 0; e < 32; ++e) zv[e] = fmaf(gC, zv[e], pv[e]);
                tmem_st32(tz + ch * 32, zv);
#pragma unroll
                for (int qq = 0; qq < 4; ++qq)
                    store_f16_chunk(sm + OFF_Z, 128, r, half * 16 + ch * 4 + qq, &zv[qq * 8]);
            }
            tmem_st_wait();
            fence_proxy_async();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[CONS_S + half]);
        }
        if (ok) {
            tc_fence_after();
            float *dst = p.Zloc + ((static_cast<size_t>(bh) * p.NS + seg) * 128 + r) * 256 + half * 128;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                float zv[32];
                tmem_ld32(tz + ch * 32, zv);
#pragma unroll
                for (int e = 0; e < 32; e += 4)
                    *reinterpret_cast<float4 *>(dst + ch * 32 + e) = make_float4(zv[e], zv[e + 1], zv[e + 2], zv[e + 3]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

// ============================================================ combine
// S_start(j+1)^T = P_j^T S_start(j)^T + S_loc(j)^T, sequential over j.  One
// CTA per (16-column slice of S^T, head), 256 threads; S_start(0) = 0, so
// S_start(1) = S_loc(0) needs no product.  P_j^T (128 x 128 fp32) is
// double-buffered in shared memory with cp.async, the copy of P_(j+1)^T in
// flight while step j is computed, and this thread's entries of S_loc(j+1)
// are loaded one step ahead too.  The product runs on warp-level tensor cores
// (mma.sync m16n8k8, tf32) in split precision: each fp32 operand x is split
// into tf32 parts hi + lo and the product accumulates hi*hi + hi*lo + lo*hi
// in fp32, close to fp32 accuracy.  Warp w owns rows 16w .. 16w+15 of the
// slice; rows are padded to 132 floats, so that the scalar fragment loads
// (8 rows x 4 columns per instruction) fall in 32 different banks, and the
// current state is kept transposed (column-major) for the B fragments.
namespace cb {
constexpr int RS = 132;  // padded row stride (floats)
constexpr uint32_t SMEM_BYTES = (2 * 128 * RS + 16 * RS) * 4;
}  // namespace cb


// x = hi + lo, both tf32 (round to nearest, ties away)
__device__ __forceinline__ void split_tf32(float x, uint32_t &hi, uint32_t &lo) {
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(hi) : "f"(x));
    const float r = x - __uint_as_float(hi);
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(lo) : "f"(r));
}
// d += a (16x8 tf32, row fragment) * b (8x8 tf32, column fragment)
__device__ __forceinline__ void mma1688_tf32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

template <bool kBwd>
__global__ void __launch_bounds__(256, 1) gdn_combine_kernel(const ScanParams p) {
    using cb::RS;
    extern __shared__ __align__(16) float csm[];
    float *PT = csm;                   // [2][128][RS]: P_j^T, row t = column t of P_j
    float *curT = csm + 2 * 128 * RS;  // [16][RS]: column c of the slice of S_start(j)^T
    const int slice = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int bh = b * p.H + h;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t4 = lane & 3;
    const int r0 = warp * 16;  // this warp's rows r0 + g and r0 + g + 8
    constexpr size_t kZ = 128 * 256;  // floats per (bh, segment) of Zloc
    const float *Z = p.Zloc + static_cast<size_t>(bh) * p.NS * kZ;
    // Backward (gradient of the state, last segment first): with X = dS^T at a segment end,
    //   X(j) = P_(j+1) X(j+1) + L(j+1),  L = the segment's local dS^T (from zero at its end),
    // the same recurrence with P_j^T read transposed, the segments taken in reverse order, L from
    // its own [NS][128][128] array and the results written for segment ends NS-2 .. 0.  Step j of
    // the loop below uses segment seg_of(j) and writes the start of step j + 1 to out_of(j + 1).
    auto seg_of = [&](int j) { return kBwd ? p.NS - 1 - j : j; };
    auto out_of = [&](int j) { return kBwd ? p.NS - 1 - j : j; };
    const float *Lsrc = kBwd ? p.Lb + static_cast<size_t>(bh) * p.NS * 128 * 128 : Z;
    constexpr int kLs = kBwd ? 128 : 256;  // row stride of L
    float *Sst = (kBwd ? p.Sb : p.Sstart) + static_cast<size_t>(bh) * p.NS * 128 * 128;
    // debug: this head's segments inside Zloc and Sstart
    if (!debug_in_bounds(p.debug, static_cast<size_t>(bh) * p.NS * kZ, static_cast<size_t>(p.NS) * kZ,
                         static_cast<size_t>(p.B) * p.H * p.NS * kZ, p.status))
        return;
    pdl_launch_dependents();
    pdl_wait();  // the transfer pass's [S_loc^T | P^T] are complete
    if (p.NS < 2) return;

    auto load_pt = [&](int j) {  // rows of P_j^T: 32 16-byte pieces each, a warp per row at a time
        const float *src = Z + seg_of(j) * kZ + 128;
        float *dst = PT + (j & 1) * 128 * RS;
#pragma unroll 4
        for (int e = tid; e < 128 * 32; e += 256) {
            const int t = e >> 5, q = e & 31;
            cp_async16(dst + t * RS + q * 4, src + static_cast<size_t>(t) * 256 + q * 4);
        }
        cp_async_commit();
    };
    // this thread's accumulator entries of S_loc(j)^T: rows r0+g (+8), columns 8n + 2t4 (+1), n = 0, 1
    auto load_sl = [&](int j, float2 (&v)[2][2]) {
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
                v[n][hh] = *reinterpret_cast<const float2 *>(Lsrc + static_cast<size_t>(seg_of(j)) * 128 * kLs +
                                                            static_cast<size_t>(r0 + g + 8 * hh) * kLs + slice * 16 +
                                                            8 * n + 2 * t4);
    };
    if (tid == 0) GDN_TRACE_AT(2048);
    if (p.NS > 2) load_pt(1);

    // S_start(1) = S_loc(0)
    for (int e = tid; e < 128 * 16; e += 256) {
        const int t = e >> 4, c = e & 15;
        const float v = Lsrc[static_cast<size_t>(seg_of(0)) * 128 * kLs + static_cast<size_t>(t) * kLs + slice * 16 + c];
        curT[c * RS + t] = v;
        Sst[(static_cast<size_t>(out_of(1)) * 128 + t) * 128 + slice * 16 + c] = v;
    }
    float2 sl[2][2];
    if (p.NS > 2) load_sl(1, sl);
    for (int j = 1; j + 1 < p.NS; ++j) {
        float2 sn[2][2];
        if (j + 2 < p.NS) {
            load_sl(j + 1, sn);
            load_pt(j + 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        if (tid == 0) GDN_TRACE_AT(2048 + 8 * j);
        __syncthreads();  // P_j^T and the current state visible to all
        if (tid == 0) GDN_TRACE_AT(2048 + 8 * j + 1);
        const float *P = PT + (j & 1) * 128 * RS;
        // three accumulators per output tile (hi*hi, hi*lo, lo*hi): independent mma chains
        float acc[2][4], ahl[2][4], alh[2][4];
#pragma unroll
        for (int n = 0; n < 2; ++n) {
            acc[n][0] = sl[n][0].x;
            acc[n][1] = sl[n][0].y;
            acc[n][2] = sl[n][1].x;
            acc[n][3] = sl[n][1].y;
#pragma unroll
            for (int e = 0; e < 4; ++e) ahl[n][e] = alh[n][e] = 0.0f;
        }
#pragma unroll 4
        for (int k0 = 0; k0 < 128; k0 += 8) {
            uint32_t ah[4], al[4];
            // A fragment: element (row, k) of P_j^T, or of P_(j+1) (the stored tile transposed)
            auto pa = [&](int row, int k) { return kBwd ? P[k * RS + row] : P[row * RS + k]; };
            split_tf32(pa(r0 + g, k0 + t4), ah[0], al[0]);
            split_tf32(pa(r0 + g + 8, k0 + t4), ah[1], al[1]);
            split_tf32(pa(r0 + g, k0 + t4 + 4), ah[2], al[2]);
            split_tf32(pa(r0 + g + 8, k0 + t4 + 4), ah[3], al[3]);
#pragma unroll
            for (int n = 0; n < 2; ++n) {
                uint32_t bh2[2], bl2[2];
                split_tf32(curT[(8 * n + g) * RS + k0 + t4], bh2[0], bl2[0]);
                split_tf32(curT[(8 * n + g) * RS + k0 + t4 + 4], bh2[1], bl2[1]);
                mma1688_tf32(alh[n], al, bh2);
                mma1688_tf32(ahl[n], ah, bl2);
                mma1688_tf32(acc[n], ah, bh2);
            }
        }
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[n][e] += ahl[n][e] + alh[n][e];
        if (tid == 0) GDN_TRACE_AT(2048 + 8 * j + 2);
        __syncthreads();  // every read of this step's state and P_j^T buffer is done
#pragma unroll
        for (int n = 0; n < 2; ++n) {
            const int c = 8 * n + 2 * t4;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int t = r0 + g + 8 * hh;
                const float v0 = acc[n][2 * hh], v1 = acc[n][2 * hh + 1];
                curT[c * RS + t] = v0;
                curT[(c + 1) * RS + t] = v1;
                *reinterpret_cast<float2 *>(Sst + (static_cast<size_t>(out_of(j + 1)) * 128 + t) * 128 + slice * 16 + c) =
                    make_float2(v0, v1);
            }
        }
        if (j + 2 < p.NS) {
#pragma unroll
            for (int n = 0; n < 2; ++n) {
                sl[n][0] = sn[n][0];
                sl[n][1] = sn[n][1];
            }
        }
        if (tid == 0) GDN_TRACE_AT(2048 + 8 * j + 3);
    }
}

// ============================================================ pass C
namespace tc {
constexpr uint32_t OFF_W = 0, OFF_QT = 32768, OFF_KT = 65536, OFF_AQK = 98304, OFF_U = 131072;
constexpr uint32_t OFF_S = 163840;  // S^T fp16 MN-major B operand (rows d_k, cols d_v)
constexpr uint32_t OFF_D = 196608;  // Delta fp16 MN-major B operand (rows token, cols d_v)
constexpr uint32_t OFF_BAR = 229376;
constexpr int NBAR = 12;
constexpr uint32_t OFF_NW = OFF_BAR + NBAR * 8 + 16;  // norm weight, fp32 [128]
constexpr uint32_t SMEM_BYTES = OFF_NW + 512 + 1024;
// One O-complete barrier per O buffer: with a single one, the producer could complete blocks i and
// i + 1 before the output warps wait for block i, whose parity wait would then alias block i + 2.
enum { FULL_WQ = 0, FULL_U, FULL_KA, MMA_X, MMA_P, MMA_O0, MMA_O1, CONS_D, CONS_S, CONS_O0, CONS_O1, TEST };
constexpr int kScanThreads = 416;  // warps 0-3 state, warp 4 producer, warps 5-12 output step
// X and P share columns (X is read out before P is written, P before the next X);
// the fp32 state S^T lives in TMEM; O is double-buffered (256 and 384).
constexpr uint32_t TM_X = 0, TM_P = 0, TM_S = 128, TM_O = 256;
}  // namespace tc

template <typename ZT>
__global__ void __launch_bounds__(tc::kScanThreads, 1)
    gdn_scan_out_kernel(const ScanParams p, const __grid_constant__ CUtensorMap tmW,
                        const __grid_constant__ CUtensorMap tmQt, const __grid_constant__ CUtensorMap tmKt,
                        const __grid_constant__ CUtensorMap tmAqk, const __grid_constant__ CUtensorMap tmAqkH,
                        const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmZ) {
    using namespace tc;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + NBAR);
    AbortState *ab = reinterpret_cast<AbortState *>(tmem_slot + 1);

    const int seg = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int bh = b * p.H + h;
    const int c0 = seg * p.Ls, c1 = min(c0 + p.Ls, p.NB);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint64_t lim = p.wait_limit_ns;

    // debug: the segment's blocks inside the [BH][Tp] tiles and gates, its start state inside Sstart
    if (!debug_in_bounds(p.debug, static_cast<size_t>(bh) * p.Tp + static_cast<size_t>(c0) * kBlk,
                         static_cast<size_t>(max(c1 - c0, 0)) * kBlk, static_cast<size_t>(p.B) * p.H * p.Tp, p.status) ||
        !debug_in_bounds(p.debug, (static_cast<size_t>(bh) * p.NS + seg) * 128 * 128, 128 * 128,
                         static_cast<size_t>(p.B) * p.H * p.NS * 128 * 128, p.status))
        return;
    float *sNW = reinterpret_cast<float *>(sm + OFF_NW);
    if (tid == 0) {
        for (int i = 0; i < NBAR; ++i)
            mbar_init(&bars[i], (i == CONS_D || i == CONS_S) ? 4 : ((i == CONS_O0 || i == CONS_O1) ? 8 : 1));
        ab->flag = 0;
        fence_mbar_init();
    }
    if (tid < kD) sNW[tid] = p.norm_w[tid];
    // Aqk's upper-right 64x64 quadrant is zero and never loaded: clear it once
    for (int e = tid; e < 64 * 128 / 16; e += kScanThreads)
        reinterpret_cast<uint4 *>(sm + OFF_AQK + 16384)[e] = make_uint4(0, 0, 0, 0);
    fence_proxy_async();
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_wait();  // the segment start states (and the UT kernel's tiles) are complete

    if (warp >= 5) {
        // ------------------------------------------ output step (warps 5-12)
        // y = o / sqrt(mean(o^2) + eps) * w * SiLU(z).  Two warps per TMEM lane quarter,
        // each for 16 rows: the accumulator is read in the 16-lane layout (a row spread
        // over a quad of lanes), and z and y move as 16-byte pieces of a row, turned into
        // and out of that layout by 4x4 transposes inside each quad, so that every warp
        // access touches 8 rows x 64 contiguous bytes instead of 32 scattered rows.
        const int q = warp & 3, part = (warp - 5) >> 2;  // a warp reads only its own TMEM lane quarter
        const int quad = lane >> 2, t0 = lane & 3;
        const int rA = q * 32 + part * 16 + quad, rB = rA + 8;  // block rows of this thread
        const uint32_t tbase = tmem + (static_cast<uint32_t>(q * 32 + part * 16) << 16);
        const ZT *z = static_cast<const ZT *>(p.z);
        for (int c = c0; c < c1; ++c) {
            const int i = c - c0;
            const int tA = c * kBlk + rA, tB = c * kBlk + rB;
            bool liveA = tA < p.T, liveB = tB < p.T;
            // input / output token of each row (the reverse scan's rows run backwards)
            const int xA = liveA ? (p.rev ? p.T - 1 - tA : tA) : 0, xB = liveB ? (p.rev ? p.T - 1 - tB : tB) : 0;
            const size_t zA = (static_cast<size_t>(b) * p.T + xA) * p.tok_stride + static_cast<size_t>(h) * kD;
            const size_t zB = (static_cast<size_t>(b) * p.T + xB) * p.tok_stride + static_cast<size_t>(h) * kD;
            const size_t yA = ((static_cast<size_t>(b) * p.T + xA) * p.H + h) * kD;
            const size_t yB = ((static_cast<size_t>(b) * p.T + xB) * p.H + h) * kD;
            if (p.debug) {  // z rows inside [B][T] x tok_stride, y rows inside [B][T][H][128]
                const size_t zsize = (static_cast<size_t>(p.B) * p.T - 1) * p.tok_stride + static_cast<size_t>(p.H) * kD;
                const size_t ysize = static_cast<size_t>(p.B) * p.T * p.H * kD;
                liveA = liveA && debug_in_bounds(1, zA, kD, zsize, p.status) && debug_in_bounds(1, yA, kD, ysize, p.status);
                liveB = liveB && debug_in_bounds(1, zB, kD, zsize, p.status) && debug_in_bounds(1, yB, kD, ysize, p.status);
            }
            const bool tre = (warp == 5 && lane == 0);
            if (tre) GDN_TRACE_AT(4096 + 64 * i + 32);
            // z: lane t0 of the quad fetches columns 8(4k + t0) .. +7 of its two rows
            uint4 za[4], zb[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int col = 8 * (4 * k + t0);
                za[k] = liveA ? *reinterpret_cast<const uint4 *>(z + zA + col) : make_uint4(0, 0, 0, 0);
                zb[k] = liveB ? *reinterpret_cast<const uint4 *>(z + zB + col) : make_uint4(0, 0, 0, 0);
            }
            if (!warp_wait(&bars[MMA_O0 + (i & 1)], (i >> 1) & 1, ab, p.status, lim)) break;
            if (tre) GDN_TRACE_AT(4096 + 64 * i + 33);
            tc_fence_after();
            const uint32_t tO = tbase + TM_O + (i & 1) * 128;
            float ssA = 0.0f, ssB = 0.0f;
            {
                uint32_t v[64];
                tmem_ld16x256b_x16(tO, v);
#pragma unroll
                for (int g = 0; g < 16; ++g) {
                    const float a0 = __uint_as_float(v[4 * g]), a1 = __uint_as_float(v[4 * g + 1]);
                    const float b0 = __uint_as_float(v[4 * g + 2]), b1 = __uint_as_float(v[4 * g + 3]);
                    ssA = fmaf(a0, a0, fmaf(a1, a1, ssA));
                    ssB = fmaf(b0, b0, fmaf(b1, b1, ssB));
                }
            }
            ssA += __shfl_xor_sync(0xffffffffu, ssA, 1);
            ssA += __shfl_xor_sync(0xffffffffu, ssA, 2);
            ssB += __shfl_xor_sync(0xffffffffu, ssB, 1);
            ssB += __shfl_xor_sync(0xffffffffu, ssB, 2);
            const float rnA = p.raw_o ? 1.0f : 1.0f / sqrtf(ssA * (1.0f / 128.0f) + p.eps);
            const float rnB = p.raw_o ? 1.0f : 1.0f / sqrtf(ssB * (1.0f / 128.0f) + p.eps);
            if (tre) GDN_TRACE_AT(4096 + 64 * i + 34);
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                uint32_t v[32];
                tmem_ld16x256b_x8(tO + hf * 64, v);  // groups g = 8hf .. 8hf+7
#pragma unroll
                for (int kk = 0; kk < 2; ++kk) {
                    const int k = 2 * hf + kk;  // groups 4k .. 4k+3
                    uint32_t wa[4] = {za[k].x, za[k].y, za[k].z, za[k].w};
                    uint32_t wb[4] = {zb[k].x, zb[k].y, zb[k].z, zb[k].w};
                    quad_transpose(wa, t0);  // wa[j] = z pair (col 8(4k+j) + 2t0, +1) of row A
                    quad_transpose(wb, t0);
                    float yf[2][4][2];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int gl = 4 * kk + j;  // group within this half
                        const int col = 8 * (4 * k + j) + 2 * t0;
                        const float w0 = sNW[col], w1 = sNW[col + 1];
                        float2 fa, fb;
                        if constexpr (sizeof(ZT) == 2 && std::is_same<ZT, __half>::value) {
                            fa = unpack_half2(wa[j]);
                            fb = unpack_half2(wb[j]);
                        } else {
                            fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&wa[j]));
                            fb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&wb[j]));
                        }
                        if (p.raw_o) {  // o itself, for the backward
                            yf[0][j][0] = __uint_as_float(v[4 * gl]);
                            yf[0][j][1] = __uint_as_float(v[4 * gl + 1]);
                            yf[1][j][0] = __uint_as_float(v[4 * gl + 2]);
                            yf[1][j][1] = __uint_as_float(v[4 * gl + 3]);
                            continue;
                        }
                        yf[0][j][0] = __uint_as_float(v[4 * gl]) * rnA * w0 * silu_tc(fa.x);
                        yf[0][j][1] = __uint_as_float(v[4 * gl + 1]) * rnA * w1 * silu_tc(fa.y);
                        yf[1][j][0] = __uint_as_float(v[4 * gl + 2]) * rnB * w0 * silu_tc(fb.x);
                        yf[1][j][1] = __uint_as_float(v[4 * gl + 3]) * rnB * w1 * silu_tc(fb.y);
                    }
                    if (p.debug) {  // every output of a live row must be finite
                        bool bad = false;
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            bad |= (liveA && !(isfinite(yf[0][j][0]) && isfinite(yf[0][j][1]))) ||
                                   (liveB && !(isfinite(yf[1][j][0]) && isfinite(yf[1][j][1])));
                        if (bad) atomicCAS(p.status, kStatusOk, kStatusCheck);
                    }
                    if (p.out_kind == 1) {  // fp32: each lane stores its 8-byte pairs (a quad covers 32 bytes)
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const int col = 8 * (4 * k + j) + 2 * t0;
                            if (liveA) *reinterpret_cast<float2 *>(static_cast<float *>(p.y) + yA + col) = make_float2(yf[0][j][0], yf[0][j][1]);
                            if (liveB) *reinterpret_cast<float2 *>(static_cast<float *>(p.y) + yB + col) = make_float2(yf[1][j][0], yf[1][j][1]);
                        }
                    } else {  // 16-bit: back to 16-byte pieces of a row, then one 16-byte store per row
                        uint32_t ya[4], yb[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            if (p.out_kind == 0) {
                                __nv_bfloat162 pa = __floats2bfloat162_rn(yf[0][j][0], yf[0][j][1]);
                                __nv_bfloat162 pb = __floats2bfloat162_rn(yf[1][j][0], yf[1][j][1]);
                                ya[j] = *reinterpret_cast<uint32_t *>(&pa);
                                yb[j] = *reinterpret_cast<uint32_t *>(&pb);
                            } else {
                                ya[j] = pack_half2(yf[0][j][0], yf[0][j][1]);
                                yb[j] = pack_half2(yf[1][j][0], yf[1][j][1]);
                            }
                        }
                        quad_transpose(ya, t0);  // ya = the 4 pairs of group 4k + t0 of row A
                        quad_transpose(yb, t0);
                        const int col = 8 * (4 * k + t0);
                        uint16_t *y16 = static_cast<uint16_t *>(p.y);
                        if (liveA) *reinterpret_cast<uint4 *>(y16 + yA + col) = make_uint4(ya[0], ya[1], ya[2], ya[3]);
                        if (liveB) *reinterpret_cast<uint4 *>(y16 + yB + col) = make_uint4(yb[0], yb[1], yb[2], yb[3]);
                    }
                }
            }
            if (tre) GDN_TRACE_AT(4096 + 64 * i + 35);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[CONS_O0 + (i & 1)]);
            if (tre) GDN_TRACE_AT(4096 + 64 * i + 36);
        }
    } else if (warp == 4) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            bool ok = true;
            const int rowbase = bh * p.Tp;
            // phases this thread has started on each barrier it feeds (TMA loads, commits), for the
            // drain below; every phase but a barrier's last is waited on before the next starts
            int started[CONS_D] = {};
            auto load2 = [&](uint32_t off, const CUtensorMap *m, uint64_t *bar, int c) {
                tma_load_2d(sm + off, m, bar, 0, rowbase + c * kBlk);
                tma_load_2d(sm + off + 16384, m, bar, 64, rowbase + c * kBlk);
            };
            auto load_wq = [&](int c) {
                ++started[FULL_WQ];
                mbar_arrive_expect_tx(&bars[FULL_WQ], 65536);
                load2(OFF_W, &tmW, &bars[FULL_WQ], c);
                load2(OFF_QT, &tmQt, &bars[FULL_WQ], c);
            };
            auto load_u = [&](int c) {
                ++started[FULL_U];
                mbar_arrive_expect_tx(&bars[FULL_U], 32768);
                load2(OFF_U, &tmU, &bars[FULL_U], c);
            };
            auto load_ka = [&](int c) {  // Kt, and Aqk but for its zero upper-right quadrant
                ++started[FULL_KA];
                mbar_arrive_expect_tx(&bars[FULL_KA], 32768 + 16384 + 8192);
                load2(OFF_KT, &tmKt, &bars[FULL_KA], c);
                tma_load_2d(sm + OFF_AQK, &tmAqk, &bars[FULL_KA], 0, rowbase + c * kBlk);
                tma_load_2d(sm + OFF_AQK + 16384 + 64 * 128, &tmAqkH, &bars[FULL_KA], 64, rowbase + c * kBlk + 64);
            };
            // first z row of block c in input order (clamped at 0; the box covers the block's rows)
            auto zrow = [&](int c) { return p.rev ? max(p.T - (c + 1) * kBlk, 0) : c * kBlk; };
            if (ok) {
                load_wq(c0);
                load_u(c0);
                load_ka(c0);
                if (c0 * kBlk < p.T) tma_prefetch_3d(&tmZ, h * kD, zrow(c0), b);
            }
            const uint32_t id_kmn = idesc_f16_f32(128, 128, false, true);
            const uint32_t id_mnmn = idesc_f16_f32(128, 128, true, true);
            for (int c = c0; ok && c < c1; ++c) {
                const int i = c - c0;
                const uint32_t ph = i & 1;
                const uint32_t tO = tmem + TM_O + (i & 1) * 128;
                if (c + 2 < c1) {  // pull the tiles of block c+2 into L2 ahead of their TMA loads
                    const int y2 = rowbase + (c + 2) * kBlk;
                    for (int hf = 0; hf < 2; ++hf) {
                        tma_prefetch_2d(&tmW, hf * 64, y2);
                        tma_prefetch_2d(&tmQt, hf * 64, y2);
                        tma_prefetch_2d(&tmU, hf * 64, y2);
                        tma_prefetch_2d(&tmKt, hf * 64, y2);
                        if (hf == 0) tma_prefetch_2d(&tmAqk, 0, y2);
                        else tma_prefetch_2d(&tmAqkH, 64, y2 + 64);
                    }
                }
                if (c + 1 < c1 && (c + 1) * kBlk < p.T)  // z rows the epilogue of block c+1 reads
                    tma_prefetch_3d(&tmZ, h * kD, zrow(c + 1), b);
                GDN_TRACE_AT(4096 + 64 * i + 0);
                ok = mbar_wait(&bars[FULL_WQ], ph, ab, p.status, lim);
                GDN_TRACE_AT(4096 + 64 * i + 1);
                ok = ok && mbar_wait(&bars[CONS_S], ph, ab, p.status, lim);
                GDN_TRACE_AT(4096 + 64 * i + 2);
                ok = ok && (i < 2 || mbar_wait(&bars[CONS_O0 + (i & 1)], ((i >> 1) - 1) & 1, ab, p.status, lim));
                GDN_TRACE_AT(4096 + 64 * i + 3);
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
                umma_commit(&bars[MMA_X]);
                ++started[MMA_X];
                GDN_TRACE_AT(4096 + 64 * i + 4);
                ok = mbar_wait(&bars[MMA_X], ph, ab, p.status, lim);
                GDN_TRACE_AT(4096 + 64 * i + 5);
                if (!ok) break;
                if (c + 1 < c1) load_wq(c + 1);
                if (p.test_wait_timeout) {
                    // test hook: mid-pipeline, with the next block's W/Qt, this block's Kt/Aqk and U in
                    // flight, a wait on a barrier nothing arrives on (bounded, ~50 ms); it sets the
                    // timeout status and the abort flag, every thread leaves its loop, and the drain
                    // below lets the loads finish before the CTA exits
                    mbar_wait(&bars[TEST], 0, ab, p.status, 50ull * 1000 * 1000);
                    ok = false;
                    break;
                }
                ok = mbar_wait(&bars[FULL_KA], ph, ab, p.status, lim);
                GDN_TRACE_AT(4096 + 64 * i + 6);
                ok = ok && mbar_wait(&bars[CONS_D], ph, ab, p.status, lim);
                GDN_TRACE_AT(4096 + 64 * i + 7);
                if (!ok) break;
                if (c + 1 < c1) load_u(c + 1);
                tc_fence_after();
                // P = Kt^T Delta  (A = Kt read MN-major: M = d_k, K = token; B = Delta MN-major)
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    umma_f16(tmem + TM_P, sdesc_sw128(sbase + OFF_KT + kk * 2048, 16384, 1024),
                             sdesc_sw128(sbase + OFF_D + kk * 2048, 16384, 1024), id_mnmn, kk > 0);
                umma_commit(&bars[MMA_P]);
                ++started[MMA_P];
                // O += Aqk Delta  (A K-major: M = token r, K = token i)
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t aoff = (kk >> 2) * 16384 + (kk & 3) * 32;
                    umma_f16(tO, sdesc_sw128(sbase + OFF_AQK + aoff, 16, 1024),
                             sdesc_sw128(sbase + OFF_D + kk * 2048, 16384, 1024), id_kmn, 1);
                }
                umma_commit(&bars[MMA_O0 + (i & 1)]);
                ++started[MMA_O0 + (i & 1)];
                GDN_TRACE_AT(4096 + 64 * i + 8);
                ok = mbar_wait(&bars[MMA_O0 + (i & 1)], (i >> 1) & 1, ab, p.status, lim);
                GDN_TRACE_AT(4096 + 64 * i + 9);
                if (!ok) break;
                if (c + 1 < c1) load_ka(c + 1);
            }
            // loads and products still in flight (after an abort) complete before shared memory and
            // TMEM go away; immediate when everything has completed
#pragma unroll 1
            for (int k = 0; k < CONS_D; ++k)
                if (started[k] > 0) mbar_wait_drain(&bars[k], (started[k] - 1) & 1, lim);
        }
    } else {
        // ----------------------------------------------------------- consumers
        const int r = tid;  // TMEM lane: token row (X) or d_k row (P, S^T)
        const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
        // initial state: S^T row r (= column r of S) into TMEM (fp32) and the fp16 operand tile
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
            float v[32];
            if (seg == 0) {
                // S^T row r = column r of the initial state (zero unless one is given)
                const float *src = p.s0 ? p.s0 + (static_cast<size_t>(bh) * 128 + ch * 32) * 128 + r : nullptr;
#pragma unroll
                for (int e = 0; e < 32; ++e) v[e] = src ? src[static_cast<size_t>(e) * 128] : 0.0f;
            } else {
                const float *src = p.Sstart + ((static_cast<size_t>(bh) * p.NS + seg) * 128 + r) * 128 + ch * 32;
#pragma unroll
                for (int e = 0; e < 32; e += 4) {
                    const float4 x = *reinterpret_cast<const float4 *>(src + e);
                    v[e] = x.x; v[e + 1] = x.y; v[e + 2] = x.z; v[e + 3] = x.w;
                }
            }
            tmem_st32(tmem + lane_base + TM_S + ch * 32, v);
            __half *g0 = p.S0b ? p.S0b + (static_cast<size_t>(bh) * p.Tp + static_cast<size_t>(c0) * kBlk + r) * 128 : nullptr;
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) store_f16_chunk2(sm + OFF_S, 128, r, ch * 4 + qq, &v[qq * 8], g0);
        }
        tmem_st_wait();
        fence_proxy_async();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[CONS_S]);

        const float *Gbh = p.G + static_cast<size_t>(bh) * p.Tp;
        bool done = true;
        for (int c = c0; c < c1; ++c) {
            done = false;
            const int i = c - c0;
            const uint32_t ph = i & 1;
            const float gC = __expf(fminf(Gbh[c * kBlk + kBlk - 1], 0.0f));
            const bool tr = (tid == 0);
            if (tr) GDN_TRACE_AT(4096 + 64 * i + 16);
            if (!warp_wait(&bars[MMA_X], ph, ab, p.status, lim)) break;
            if (tr) GDN_TRACE_AT(4096 + 64 * i + 17);
            if (!warp_wait(&bars[FULL_U], ph, ab, p.status, lim)) break;
            if (tr) GDN_TRACE_AT(4096 + 64 * i + 18);
            tc_fence_after();
            // Delta = U - X, row r
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                float x[32];
                tmem_ld32(tmem + lane_base + TM_X + ch * 32, x);
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    const uint4 uu = *reinterpret_cast<const uint4 *>(sm + OFF_U + tile_off(128, r, ch * 4 + qq));
                    const uint32_t w4[4] = {uu.x, uu.y, uu.z, uu.w};
                    float dlt[8];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 u2 = unpack_half2(w4[e]);
                        dlt[2 * e] = u2.x - x[qq * 8 + 2 * e];
                        dlt[2 * e + 1] = u2.y - x[qq * 8 + 2 * e + 1];
                    }
                    store_f16_chunk(sm + OFF_D, 128, r, ch * 4 + qq, dlt);
                }
            }
            fence_proxy_async();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[CONS_D]);
            if (tr) GDN_TRACE_AT(4096 + 64 * i + 19);

            // S^T row r <- gC * S^T row r + P row r  (state in TMEM, fp16 copy for the next MMAs)
            if (!warp_wait(&bars[MMA_P], ph, ab, p.status, lim)) break;
            if (tr) GDN_TRACE_AT(4096 + 64 * i + 20);
            tc_fence_after();
            // the state at the start of block c + 1, kept for the backward
            __half *gs = (p.S0b && c + 1 < c1)
                             ? p.S0b + (static_cast<size_t>(bh) * p.Tp + static_cast<size_t>(c + 1) * kBlk + r) * 128
                             : nullptr;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                float pv[32], sv[32];
                tmem_ld32(tmem + lane_base + TM_P + ch * 32, pv);
                tmem_ld32(tmem + lane_base + TM_S + ch * 32, sv);
#pragma unroll
                for (int e = 0; e < 32; ++e) sv[e] = fmaf(gC, sv[e], pv[e]);
                tmem_st32(tmem + lane_base + TM_S + ch * 32, sv);
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) store_f16_chunk2(sm + OFF_S, 128, r, ch * 4 + qq, &sv[qq * 8], gs);
            }
            tmem_st_wait();
            fence_proxy_async();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[CONS_S]);
            if (tr) GDN_TRACE_AT(4096 + 64 * i + 21);
            done = true;
        }
        if (done && p.s_end && seg == p.NS - 1) {
            // the state after the last block (padding tokens leave it unchanged): S^T row r is
            // column r of S; a warp's 32 lanes write 32 consecutive floats of each row of S
            float *dst = p.s_end + (static_cast<size_t>(bh) * 128) * 128 + r;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                float sv[32];
                tmem_ld32(tmem + lane_base + TM_S + ch * 32, sv);
#pragma unroll
                for (int e = 0; e < 32; ++e) dst[static_cast<size_t>(ch * 32 + e) * 128] = sv[e];
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 512);
}


}  // namespace

cudaError_t launch_transfer(const ScanParams &p, const CUtensorMap &tmW, const CUtensorMap &tmKt,
                            const CUtensorMap &tmU, cudaStream_t s, bool pdl) {
    static SmemOnce once;
    cudaError_t e = raise_smem_once(once, gdn_transfer_kernel, static_cast<int>(ta::SMEM_BYTES));
    if (e != cudaSuccess) return e;
    dim3 grid(p.NS - 1, p.H, p.B);
    return launch_k(gdn_transfer_kernel, grid, dim3(288), ta::SMEM_BYTES, s, pdl, p, tmW, tmKt, tmU);
}

cudaError_t launch_combine(const ScanParams &p, cudaStream_t s, bool pdl) {
    static SmemOnce once;
    cudaError_t e = raise_smem_once(once, gdn_combine_kernel<false>, static_cast<int>(cb::SMEM_BYTES));
    if (e != cudaSuccess) return e;
    dim3 grid(8, p.H, p.B);
    return launch_k(gdn_combine_kernel<false>, grid, dim3(256), cb::SMEM_BYTES, s, pdl, p);
}

cudaError_t launch_combine_bwd(const ScanParams &p, cudaStream_t s, bool pdl) {
    static SmemOnce once;
    cudaError_t e = raise_smem_once(once, gdn_combine_kernel<true>, static_cast<int>(cb::SMEM_BYTES));
    if (e != cudaSuccess) return e;
    dim3 grid(8, p.H, p.B);
    return launch_k(gdn_combine_kernel<true>, grid, dim3(256), cb::SMEM_BYTES, s, pdl, p);
}

cudaError_t launch_scan_out(const ScanParams &p, InType zt, const CUtensorMap &tmW, const CUtensorMap &tmQt,
                            const CUtensorMap &tmKt, const CUtensorMap &tmAqk, const CUtensorMap &tmAqkH,
                            const CUtensorMap &tmU, const CUtensorMap &tmZ, cudaStream_t s, bool pdl) {
    dim3 grid(p.NS, p.H, p.B);
    if (zt == InType::F16) {
        static SmemOnce once;
        cudaError_t e = raise_smem_once(once, gdn_scan_out_kernel<__half>, static_cast<int>(tc::SMEM_BYTES));
        if (e != cudaSuccess) return e;
        return launch_k(gdn_scan_out_kernel<__half>, grid, dim3(tc::kScanThreads), tc::SMEM_BYTES, s, pdl, p, tmW,
                        tmQt, tmKt, tmAqk, tmAqkH, tmU, tmZ);
    }
    static SmemOnce once;
    cudaError_t e = raise_smem_once(once, gdn_scan_out_kernel<__nv_bfloat16>, static_cast<int>(tc::SMEM_BYTES));
    if (e != cudaSuccess) return e;
    return launch_k(gdn_scan_out_kernel<__nv_bfloat16>, grid, dim3(tc::kScanThreads), tc::SMEM_BYTES, s, pdl, p, tmW,
                    tmQt, tmKt, tmAqk, tmAqkH, tmU, tmZ);
}

}  // namespace gdn

GDN_TRACE_EXPORT(scan)
