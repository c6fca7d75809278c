// gdn_fused.cu -- the GDN forward on the tensor path (d_k = d_v = 128, 16-bit
// inputs): the gated delta rule of "Gated Delta Networks: Improving Mamba2 with
// Delta Rule" (reference [57] on the VMonarch page) with the per-token parts the
// LinMorph page lists ("Why learn the initialization?": short convolutions,
// normalization, decay terms, update gates), as two fused persistent passes over
// segments of the sequence and a combine of the segment states.
//
// Per block of C = 64 tokens (the UT chunk), with G_r the in-block cumulative
// log decay and incoming state S (d_v x d_k):
//   L_rj = beta_r e^(G_r-G_j) k_r.k_j (j < r),  T = (I + L)^-1,
//   U^T  = V^T (T diag(beta))^T,  W^T = K^T (T diag(beta e^G))^T,
//   Delta^T = U^T - S W^T,
//   O^T  = S (diag(e^G) Q)^T + Delta^T Aqk^T,  Aqk_ri = [i <= r] e^(G_r-G_i) q_r.k_i,
//   S   <- e^(G_C) S + Delta^T diag(e^(G_C-G)) K.
// Every product has M = 128 in this transposed form (rows of S, or of K^T, V^T
// for W^T, U^T), so all of them run as tcgen05 kind::f16 MMAs with the fp32
// accumulators in tensor memory, one TMEM lane per row of the state.  The state
// is kept negated (N = -S) so that Delta^T = U^T + N W^T is a plain
// accumulation into the U^T columns; its fp16 copy N16 and the fp16 Delta (E16
// = -Delta^T) are MMA A operands read straight from tensor memory.
//
// Nothing of a block but its raw inputs crosses HBM.  Each CTA owns one segment
// of one (b, h) and walks its blocks in order; warp groups overlap the next
// block's preparation and UT transform with the current block's state step:
//   warp 0       MMA issue (one thread)
//   warps 1-4    prep: raw q/k/v boxes (64 tokens + 3 of conv history) by TMA,
//                conv4 + SiLU (+ L2 norm for q, k; the 1/sqrt(d_k) output scale
//                folded into q) into fp16 operand tiles
//   warps 5-8    gates, L and Aqk from the stacked Gram [K; Q] K^T, the blocked
//                inverse (I + L)^-1, the scaled T tiles, W^T out of TMEM, Qt, Kt
//   warps 9-12   the state step (lanes = rows of S)
//   warps 13-16  output pass: the output step y = o/sqrt(mean(o^2)+eps) w SiLU(z)
//                (z in and y out by TMA); transfer pass: the transfer matrix
// The transfer pass (kOut = false) runs every segment but the last from S = 0
// (or the given initial state for segment 0) next to the transfer matrix P
// from I, and writes S_loc and P; gdn_combine_kernel chains
// S_start(j+1) = S_start(j) P_j + S_loc(j) in fp32; the output pass (kOut =
// true) reruns every segment from its start state and writes y.
//
// Every hand-off is an mbarrier with a bounded wait.  A wait that runs out sets
// the device status word and the CTA's abort flag; every role then leaves its
// loop, and before tensor memory is released the MMA thread waits (bounded) for
// the tensor-core work it issued and each TMA thread for the loads and stores
// it issued.  No TMA multicast is used.
#include <type_traits>

#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

// timeline stamp k of block i (compiled in only for tuning builds, see GDN_TRACE)
#define FTRACE(i, k) GDN_TRACE_AT((kOut ? 0 : 4096) + (i) * 32 + (k))

constexpr int kC = 64;                      // tokens per block
constexpr int kRawRows = kC + 3;            // conv window: 3 tokens of history
constexpr uint32_t kRawBytes = kRawRows * 256;  // one raw box: 67 tokens x 128 channels x 16 bit
constexpr int kThreads = 544;               // 17 warps
enum { W_MMA = 0, W_PREP = 1, W_UT = 5, W_CH = 9, W_X = 13 };  // first warp of each role
enum { NB_PREP = 1, NB_UT = 2, NB_X = 3 };                      // named barriers (128 threads)

// Shared-memory map (offsets from a 1024-byte aligned base).  The KQ, W^T, Aqk, T and TW
// tiles come in two slots (block i uses slot i & 1), so that the next block's UT transform
// runs while the current block's state step reads its operands.
template <bool kOut>
struct Lay;
template <>
struct Lay<true> {  // output pass
    static constexpr uint32_t KQ = 0;        // 2 x [128 rows: K' (0-63) -> Kt, Q' (64-127) -> Qt][128] fp16
    static constexpr uint32_t WT = 65536;    // 2 x W^T [128 d_k][64 tokens] fp16
    static constexpr uint32_t AQK = 98304;   // 2 x Aqk [64][64] fp16
    static constexpr uint32_t V = 114688;    // V' [64][128] fp16
    static constexpr uint32_t T = 131072;    // 2 x (L -> T -> T diag(beta)) [64][64] fp16
    static constexpr uint32_t TW = 147456;   // 2 x T diag(beta e^G / |k'|) [64][64] fp16
    static constexpr uint32_t RAW = 163840;  // 2 raw-box slots; the block's k, q, v boxes rotate through them
    static constexpr uint32_t Z = 198144;    // z box [64][128] 16-bit, y written over it
    static constexpr uint32_t MISC = 214528;
    static constexpr int NRAWSLOT = 2, NTENS = 3;
};
template <>
struct Lay<false> {  // transfer pass
    static constexpr uint32_t KQ = 0;        // 2 x [128 rows: K' (0-63) -> Kt, V' (64-127)][128] fp16
    static constexpr uint32_t WT = 65536;
    static constexpr uint32_t N16S = 98304;  // fp16 copy of -S, A operand [128][128] K-major
    static constexpr uint32_t N16P = 131072; // fp16 copy of -P
    static constexpr uint32_t T = 163840;
    static constexpr uint32_t TW = 180224;
    static constexpr uint32_t RAW = 196608;  // one raw-box slot: the block's k, then v
    static constexpr uint32_t MISC = 213760;
    static constexpr int NRAWSLOT = 1, NTENS = 2;
};
// MISC sub-layout
constexpr uint32_t M_GATE = 0;      // 2 slots x {G, beta, ec, beta e^G / |k'|} x 64 fp32
constexpr uint32_t M_INVN = 2048;   // 2 slots x {1/|k'|, 1/(sqrt(d) |q'|)} x 64 fp32 (prep)
constexpr uint32_t M_LDIAG = 3072;  // the diagonal 16x16 blocks of L, fp32 [4][16][16]
constexpr uint32_t M_RED = 7168;    // output step: per-token partial sums of squares [64][4]
constexpr uint32_t M_RN = 8192;     // per-token 1/rms [64]
constexpr uint32_t M_NW = 8448;     // norm weight [128]
constexpr uint32_t M_WTOT = 8960;   // gate scan: warp totals
constexpr uint32_t M_CONV = 8992;   // conv taps of the CTA's head: [tensor][j][cg] float4, channel 8 cg + j
constexpr uint32_t M_BAR = M_CONV + 3 * 128 * 16;
constexpr int NBAR = 28;
constexpr uint32_t M_SLOT = M_BAR + NBAR * 8;  // TMEM base address, abort flag
constexpr uint32_t M_SIZE = M_SLOT + 16;
template <bool kOut>
constexpr uint32_t smem_bytes() { return Lay<kOut>::MISC + M_SIZE + 1024; }
static_assert(smem_bytes<true>() <= 227 * 1024 && smem_bytes<false>() <= 227 * 1024, "shared memory");
static_assert(Lay<true>::RAW + 2 * kRawBytes <= Lay<true>::Z && Lay<true>::Z + 16384 <= Lay<true>::MISC, "layout");
static_assert(Lay<false>::RAW + kRawBytes <= Lay<false>::MISC, "layout");

// mbarriers; "2:" = one per slot (block i uses slot i & 1), so that a waiter that runs a block
// ahead or behind never mistakes one block's phase for another's
enum {
    B_RAW = 0,         // 2: raw-box slot landed (TMA)
    B_PREP = 2,        // 2: K', Q' tiles (transfer pass: K', V') and their inverse norms complete (4 prep warps)
    B_PREPV = 4,       // output pass: the V' tile is complete (4 prep warps)
    B_FREE = 5,        // 2: every MMA that reads the slot's tiles is complete (commit)
    B_VFREE = 7,       // U^T read the V' tile (commit)
    B_GRAM = 8,        // Gram complete (commit)
    B_GATE = 9,        // 2: gates of the slot in shared memory (4 UT warps)
    B_TREADY = 11,     // 2: T tiles, Qt and Aqk of the slot complete (4 UT warps)
    B_WT = 13,         // 2: W^T and U^T of the slot complete (commit)
    B_UTD = 15,        // 2: W^T tile and Kt of the slot complete (4 state warps)
    B_DELTA = 17,      // Delta^T (and the first half of O^T) complete (commit)
    B_E16 = 18,        // fp16 Delta in TMEM (state warps)
    B_STATE = 19,      // state update complete (commit)
    B_N16 = 20,        // fp16 state copy ready, state decayed by the next block's decay (state warps)
    B_OFULL = 21,      // 2: O^T buffer complete (commit)
    B_OFREE = 23,      // 2: O^T buffer read (4 output warps)
    B_Z = 25,          // z box landed
    B_TEST = 26,       // never completes (test hook)
    B_DRAIN = 27       // teardown: every MMA issued so far is complete (commit)
};

// TMEM columns (512 allocated).  The fp16 Delta (E16) is written over the first 32 columns of
// the fp32 Delta^T it comes from.
template <bool kOut>
struct Tm;
template <>
struct Tm<true> {
    static constexpr uint32_t N = 0, N16 = 128, UD = 192, E16 = 192, GA = 256, GB = 320, O = 384;  // O: 2 x 64
};
template <>
struct Tm<false> {
    static constexpr uint32_t N = 0, NP = 128, UD = 256, UDP = 320, E16 = 256, E16P = 320, GA = 384, GB = 448;
};

// 8 consecutive 16-bit inputs -> fp32
template <typename InT>
__device__ __forceinline__ void load8(const uint8_t *p, float (&f)[8]) {
    const uint4 u = *reinterpret_cast<const uint4 *>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 x;
        if constexpr (std::is_same<InT, __half>::value) {
            x = unpack_half2(w[i]);
        } else {
            x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[i]));
        }
        f[2 * i] = x.x;
        f[2 * i + 1] = x.y;
    }
}
__device__ __forceinline__ float load1(const uint8_t *p, bool half) {
    const uint16_t u = *reinterpret_cast<const uint16_t *>(p);
    if (half) return __half2float(__ushort_as_half(u));
    return __bfloat162float(__ushort_as_bfloat16(u));
}

__device__ __forceinline__ void put8h(uint8_t *tile, int rows, int r, int chunk, const float *v) {
    uint4 u;
    u.x = pack_half2(v[0], v[1]);
    u.y = pack_half2(v[2], v[3]);
    u.z = pack_half2(v[4], v[5]);
    u.w = pack_half2(v[6], v[7]);
    *reinterpret_cast<uint4 *>(tile + tile_off(rows, r, chunk)) = u;
}
// Row r of a panel tile scaled in place by f, chunks [ch0, ch0 + nch).
__device__ __forceinline__ void scale_row_chunks(uint8_t *tile, int rows, int r, int ch0, int nch, float f) {
#pragma unroll 2
    for (int c = ch0; c < ch0 + nch; ++c) {
        uint4 *pu = reinterpret_cast<uint4 *>(tile + tile_off(rows, r, c));
        const uint4 u = *pu;
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 x = unpack_half2(w[e]);
            o[e] = pack_half2(x.x * f, x.y * f);
        }
        *pu = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// warp-level tensor-core products for the blocked inverse
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr)
                 : "memory");
}
__device__ __forceinline__ void ldsm_x2_trans(uint32_t addr, uint32_t (&r)[2]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];"
                 : "=r"(r[0]), "=r"(r[1])
                 : "r"(addr)
                 : "memory");
}
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// T = (I + L)^-1 for the 64x64 unit lower-triangular system held in the L tile (fp16, one
// 64-row panel, strict lower part; the diagonal 16x16 blocks also in fp32 in ldiag), by block
// forward substitution over the 4 x 4 grid of 16x16 blocks: D_b = (I + L_bb)^-1 by column
// solves, M_ik = D_i L_ik (k < i), then block rows T_ij = -sum_{k=j}^{i-1} M_ik T_kj.  Run by
// the 128 threads of the UT group (ut = 0..127); T overwrites the tile.
__device__ __forceinline__ void invert_unit_lower64(uint8_t *Tt, const float *ldiag, int ut) {
    const uint32_t tT = smem_u32(Tt);
    const int warp = ut >> 5, lane = ut & 31;
    if (ut < 64) {  // column c of D_b, b = ut / 16
        const int b = ut >> 4, c = ut & 15;
        const float *Lb = ldiag + b * 256;
        float x[16];
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) x[rr] = (rr == c) ? 1.0f : 0.0f;
#pragma unroll
        for (int rr = 1; rr < 16; ++rr) {
            float s0 = 0.0f, s1 = 0.0f;
#pragma unroll
            for (int k = 0; k < rr; k += 4) {
                const float4 l4 = *reinterpret_cast<const float4 *>(Lb + rr * 16 + k);
                s0 = fmaf(l4.x, x[k], s0);
                if (k + 1 < rr) s1 = fmaf(l4.y, x[k + 1], s1);
                if (k + 2 < rr) s0 = fmaf(l4.z, x[k + 2], s0);
                if (k + 3 < rr) s1 = fmaf(l4.w, x[k + 3], s1);
            }
            if (rr > c) x[rr] = -(s0 + s1);
        }
#pragma unroll
        for (int rr = 0; rr < 16; ++rr)
            *reinterpret_cast<__half *>(Tt + tile_elem_off(64, 16 * b + rr, 16 * b + c)) = __float2half_rn(x[rr]);
    }
    named_sync(NB_UT, 128);
    const int g = lane >> 2, t4 = lane & 3;
    const int lm = lane >> 3, lr = lane & 7;
    const int arow = (lm & 1) * 8 + lr, achk = lm >> 1;
    // M_ik = D_i L_ik for the six blocks below the diagonal, over L_ik
    for (int qb = warp; qb < 6; qb += 4) {
        const int i = qb < 1 ? 1 : (qb < 3 ? 2 : 3);
        const int k = qb - (i * (i - 1)) / 2;
        uint32_t a[4], b0[2], b1[2];
        ldsm_x4(tT + tile_off(64, 16 * i + arow, 2 * i + achk), a);
        ldsm_x2_trans(tT + tile_off(64, 16 * i + arow, 2 * k), b0);
        ldsm_x2_trans(tT + tile_off(64, 16 * i + arow, 2 * k + 1), b1);
        float o0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, o1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        mma16816(o0, a, b0);
        mma16816(o1, a, b1);
        __syncwarp();
        const int col = 16 * k + 2 * t4;
        *reinterpret_cast<uint32_t *>(Tt + tile_elem_off(64, 16 * i + g, col)) = pack_half2(o0[0], o0[1]);
        *reinterpret_cast<uint32_t *>(Tt + tile_elem_off(64, 16 * i + g + 8, col)) = pack_half2(o0[2], o0[3]);
        *reinterpret_cast<uint32_t *>(Tt + tile_elem_off(64, 16 * i + g, col + 8)) = pack_half2(o1[0], o1[1]);
        *reinterpret_cast<uint32_t *>(Tt + tile_elem_off(64, 16 * i + g + 8, col + 8)) = pack_half2(o1[2], o1[3]);
    }
    named_sync(NB_UT, 128);
    // block rows i = 1..3: the 2i 16x8 halves (j = q / 2, column half q % 2) over the four warps
#pragma unroll 1
    for (int i = 1; i < 4; ++i) {
        float acc[2][4];
#pragma unroll
        for (int sl = 0; sl < 2; ++sl) acc[sl][0] = acc[sl][1] = acc[sl][2] = acc[sl][3] = 0.0f;
#pragma unroll 1
        for (int k = 0; k < i; ++k) {
            uint32_t a[4];
            ldsm_x4(tT + tile_off(64, 16 * i + arow, 2 * k + achk), a);
#pragma unroll
            for (int sl = 0; sl < 2; ++sl) {
                const int q = warp + 4 * sl;
                if (q < 2 * i && (q >> 1) <= k) {
                    uint32_t bq[2];
                    ldsm_x2_trans(tT + tile_off(64, 16 * k + arow, q), bq);
                    mma16816(acc[sl], a, bq);
                }
            }
        }
        named_sync(NB_UT, 128);
#pragma unroll
        for (int sl = 0; sl < 2; ++sl) {
            const int q = warp + 4 * sl;
            if (q < 2 * i) {
                const int col = 16 * (q >> 1) + 8 * (q & 1) + 2 * t4;
                *reinterpret_cast<uint32_t *>(Tt + tile_elem_off(64, 16 * i + g, col)) =
                    pack_half2(-acc[sl][0], -acc[sl][1]);
                *reinterpret_cast<uint32_t *>(Tt + tile_elem_off(64, 16 * i + g + 8, col)) =
                    pack_half2(-acc[sl][2], -acc[sl][3]);
            }
        }
        named_sync(NB_UT, 128);
    }
}

template <bool kOut, typename InT>
__global__ void __launch_bounds__(kThreads, 1)
    gdn_fused_kernel(const FusedParams p, const __grid_constant__ CUtensorMap tmq,
                     const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                     const __grid_constant__ CUtensorMap tmz, const __grid_constant__ CUtensorMap tmy,
                     const __grid_constant__ CUtensorMap tmy_tail) {
    using Ly = Lay<kOut>;
    using TM = Tm<kOut>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    uint8_t *misc = sm + Ly::MISC;
    float *gate = reinterpret_cast<float *>(misc + M_GATE);
    float *ldiag = reinterpret_cast<float *>(misc + M_LDIAG);
    float *invn = reinterpret_cast<float *>(misc + M_INVN);
    float4 *convs = reinterpret_cast<float4 *>(misc + M_CONV);
    float *red = reinterpret_cast<float *>(misc + M_RED);
    float *rns = reinterpret_cast<float *>(misc + M_RN);
    float *nw = reinterpret_cast<float *>(misc + M_NW);
    float *wtot = reinterpret_cast<float *>(misc + M_WTOT);
    uint64_t *bars = reinterpret_cast<uint64_t *>(misc + M_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(misc + M_SLOT);
    AbortState *ab = reinterpret_cast<AbortState *>(misc + M_SLOT + 4);

    const int seg = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int bh = b * p.H + h;
    const int c0 = seg * p.Ls, c1 = min(c0 + p.Ls, p.NB), n = c1 - c0;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint64_t lim = p.wait_limit_ns;

    if (tid == 0) {
        for (int i = 0; i < NBAR; ++i) {
            int cnt = 1;  // TMA and tensor-core commits
            if ((i >= B_PREP && i < B_FREE) || (i >= B_GATE && i < B_WT) || i == B_UTD || i == B_UTD + 1 ||
                i == B_OFREE || i == B_OFREE + 1)
                cnt = 4;  // one arrival per warp of a 4-warp group
            if (i == B_E16 || i == B_N16) cnt = kOut ? 4 : 8;  // the state warps (and the transfer warps)
            mbar_init(&bars[i], cnt);
        }
        ab->flag = 0;
        fence_mbar_init();
    }
    if (kOut && tid < kD) nw[tid] = p.norm_w[tid];
    if (warp == W_MMA) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    pdl_launch_dependents();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (p.debug && tid == 0 && ((tmem & 0xFFFFu) != 0u || n < 1 || c1 > p.NB)) {
        atomicCAS(p.status, kStatusOk, kStatusCheck);
        ab->flag = 1;
    }
    __syncthreads();
    if (ab->flag) goto teardown;

    if (warp == W_MMA) {
        // ================================================================ MMA issue (one thread)
        if (lane == 0) {
            bool issued = false;
            auto kq = [&](int s) { return sb + Ly::KQ + static_cast<uint32_t>(s) * 32768u; };
            auto wtile = [&](int s) { return sb + Ly::WT + static_cast<uint32_t>(s) * 16384u; };
            const uint32_t id_kk64 = idesc_f16_f32(128, 64, false, false);   // Gram, Qt^T, Aqk^T
            const uint32_t id_mk64 = idesc_f16_f32(128, 64, true, false);    // W^T, U^T
            const uint32_t id_km64 = idesc_f16_f32(128, 64, false, true);    // Delta^T (B = W^T)
            const uint32_t id_km128 = idesc_f16_f32(128, 128, false, true);  // state (B = Kt)
            // byte offset of K-step kk (16 elements) in a K-major tile whose 64-element panels are
            // `panel` bytes apart
            auto kmaj = [](int kk, uint32_t panel) { return static_cast<uint32_t>(kk >> 2) * panel + (kk & 3) * 32u; };
            // the stacked Gram [K'; Q'] K'^T (transfer pass: [K'; V'] K'^T, lanes 64-127 unused) of block j
            auto gram = [&](int j) {
                const int s = j & 1;
#pragma unroll 1
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t d = sdesc_sw128(kq(s) + kmaj(kk, 16384), 16, 1024);
                    umma_f16(tmem + TM::GA, d, d, id_kk64, kk > 0);
                }
                umma_commit(&bars[B_GRAM]);
            };
            // W^T = K'^T (T diag(beta e^G / |k'|))^T and U^T = V'^T (T diag(beta))^T of block j
            // (output pass: U^T once the V' tile is complete)
            auto wt_ut = [&](int j) -> bool {
                const int s = j & 1;
                const uint32_t tt = sb + Ly::T + s * 8192u, tw = sb + Ly::TW + s * 8192u;
#pragma unroll 1
                for (int kk = 0; kk < 4; ++kk)
                    umma_f16(tmem + TM::GB, sdesc_sw128(kq(s) + kk * 2048, 16384, 1024),
                             sdesc_sw128(tw + kk * 32, 16, 1024), id_mk64, kk > 0);
                if (kOut) {
                    if (!mbar_wait_ol(&bars[B_PREPV], j & 1, ab, p.status, lim)) return false;
                    tc_fence_after();
                }
#pragma unroll 1
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t ad = kOut ? sdesc_sw128(sb + Lay<true>::V + kk * 2048, 8192, 1024)
                                             : sdesc_sw128(kq(s) + 8192 + kk * 2048, 16384, 1024);
                    umma_f16(tmem + TM::UD, ad, sdesc_sw128(tt + kk * 32, 16, 1024), id_mk64, kk > 0);
                }
                umma_commit(&bars[B_WT + s]);
                if (kOut) umma_commit(&bars[B_VFREE]);
                return true;
            };
            // The Gram of block j needs its prepared tiles and the Gram columns free: block j - 1's
            // L and Aqk are out once its T tiles are (TREADY).  `gram_next` is the next block whose
            // Gram is to be issued, `tready_seen` the last block whose TREADY this thread has waited for.
            int gram_next = 0, tready_seen = -1;
            auto try_gram = [&](bool block) -> bool {
                while (gram_next < n && tready_seen >= gram_next - 1) {
                    const int j = gram_next, s = j & 1;
                    if (block) {
                        if (!mbar_wait_ol(&bars[B_PREP + s], (j >> 1) & 1, ab, p.status, lim)) return false;
                    } else if (!mbar_try_wait(&bars[B_PREP + s], (j >> 1) & 1)) {
                        return true;
                    }
                    tc_fence_after();
                    gram(j);
                    issued = true;
                    if (j == 0) FTRACE(0, 5);
                    ++gram_next;
                    if (!block) break;
                    block = false;
                }
                return true;
            };
            bool ok = try_gram(true);
            ok = ok && mbar_wait_ol(&bars[B_TREADY], 0, ab, p.status, lim);
            if (ok) {
                tready_seen = 0;
                tc_fence_after();
                ok = wt_ut(0);
            }
            if (ok && p.test_timeout) {
                // test hook: a wait on a barrier nothing arrives on (bounded, ~50 ms), with tensor-core
                // work and raw loads in flight; the drains at the end let them finish
                mbar_wait_ol(&bars[B_TEST], 0, ab, p.status, 50ull * 1000 * 1000);
                ok = false;
            }
            ok = ok && try_gram(false);
            for (int i = 0; ok && i < n; ++i) {
                const int s = i & 1;
                FTRACE(i, 0);
                ok = mbar_wait_ol(&bars[B_UTD + s], (i >> 1) & 1, ab, p.status, lim) &&
                     mbar_wait_ol(&bars[B_N16], i & 1, ab, p.status, lim) &&
                     (!kOut || i < 2 || mbar_wait_ol(&bars[B_OFREE + s], ((i >> 1) - 1) & 1, ab, p.status, lim));
                if (!ok) break;
                FTRACE(i, 1);
                tc_fence_after();
                // Delta^T = U^T + N W^T (and the first half of O^T = -(S Qt^T))
#pragma unroll 1
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t bd = sdesc_sw128(wtile(s) + kk * 2048, 8192, 1024);
                    if constexpr (kOut) {
                        umma_f16_ts(tmem + TM::UD, tmem + Tm<true>::N16 + kk * 8, bd, id_km64, 1);
                        umma_f16_ts(tmem + Tm<true>::O + s * 64, tmem + Tm<true>::N16 + kk * 8,
                                    sdesc_sw128(kq(s) + 8192 + kmaj(kk, 16384), 16, 1024), id_kk64, kk > 0);
                    } else {
                        const uint32_t ao = kmaj(kk, 16384);
                        umma_f16(tmem + TM::UD, sdesc_sw128(sb + Lay<false>::N16S + ao, 16, 1024), bd, id_km64, 1);
                        umma_f16(tmem + Tm<false>::UDP, sdesc_sw128(sb + Lay<false>::N16P + ao, 16, 1024), bd, id_km64,
                                 kk > 0);
                    }
                }
                umma_commit(&bars[B_DELTA]);
                FTRACE(i, 2);
                ok = try_gram(false);
                ok = ok && mbar_wait_ol(&bars[B_E16], i & 1, ab, p.status, lim);
                if (!ok) break;
                FTRACE(i, 3);
                tc_fence_after();
                // N += E16 Kt  (E16 = -Delta^T, fp16 in TMEM; Kt MN-major, N = d_k)
#pragma unroll 1
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t bd = sdesc_sw128(kq(s) + kk * 2048, 16384, 1024);
                    umma_f16_ts(tmem + TM::N, tmem + TM::E16 + kk * 8, bd, id_km128, 1);
                    if constexpr (!kOut) umma_f16_ts(tmem + Tm<false>::NP, tmem + Tm<false>::E16P + kk * 8, bd, id_km128, 1);
                }
                umma_commit(&bars[B_STATE]);
                if constexpr (kOut) {
                    // O^T += E16 Aqk^T
                    const uint32_t aq = sb + Lay<true>::AQK + static_cast<uint32_t>(s) * 8192u;
#pragma unroll 1
                    for (int kk = 0; kk < 4; ++kk)
                        umma_f16_ts(tmem + Tm<true>::O + s * 64, tmem + TM::E16 + kk * 8,
                                    sdesc_sw128(aq + kk * 32, 16, 1024), id_kk64, 1);
                    umma_commit(&bars[B_OFULL + s]);
                }
                umma_commit(&bars[B_FREE + s]);
                FTRACE(i, 4);
                if (i + 1 < n) {
                    // the next block's W^T and U^T (its Gram first, if it is still to be issued); U^T goes
                    // to the Delta^T columns, whose fp16 Delta the state update above has read
                    ok = (gram_next > i + 1 || try_gram(true)) &&
                         mbar_wait_ol(&bars[B_TREADY + (s ^ 1)], ((i + 1) >> 1) & 1, ab, p.status, lim);
                    if (!ok) break;
                    tready_seen = i + 1;
                    FTRACE(i, 6);
                    tc_fence_after();
                    ok = wt_ut(i + 1) && try_gram(false);
                }
            }
            if (issued) {  // every tensor-core operation issued so far has completed
                umma_commit(&bars[B_DRAIN]);
                mbar_wait_drain(&bars[B_DRAIN], 0, lim);
            }
        }
    } else if (warp < W_UT) {
        // ================================================================ prep
        // conv4 + SiLU of the block's raw boxes into fp16 operand tiles.  q' and k' are stored as
        // they are; the inverse norms 1/|k'| and 1/(sqrt(d_k) |q'|) of every token go to shared
        // memory and are applied where the tiles are scaled or read next (L, Aqk, Qt, Kt, and the
        // columns of T diag(beta e^G)), so that no per-token reduction sits between a token's
        // conv and its store.  Thread (cg, rg) owns channels 8 cg .. 8 cg + 7 of tokens
        // 8 rg .. 8 rg + 7.  The raw boxes are loads number l = NTENS i + w (tensor w of block i),
        // through slot l % NRAWSLOT; load l + NRAWSLOT is issued once load l has been read.
        const int pt = tid - 32 * W_PREP;
        const int cg = pt & 15, rg = pt >> 4, rbeg = rg * 8;
        constexpr int NT = Ly::NTENS, NSL = Ly::NRAWSLOT;
        // output pass: k, q (-> Gram), then v; transfer pass: k, v
        auto map_of = [&](int w) -> const CUtensorMap * {
            if constexpr (kOut) return w == 0 ? &tmk : (w == 1 ? &tmq : &tmv);
            else return w == 0 ? &tmk : &tmv;
        };
        auto conv_of = [&](int w) -> const float * {
            if constexpr (kOut) return w == 0 ? p.conv_k : (w == 1 ? p.conv_q : p.conv_v);
            else return w == 0 ? p.conv_k : p.conv_v;
        };
        auto row0 = [&](int c) { return p.rev ? p.T - kC - c * kC : c * kC - 3; };
        const int nload = n * NT;
        auto issue = [&](int l) {  // thread 0
            const int sl = l % NSL, i = l / NT, w = l % NT;
            mbar_arrive_expect_tx(&bars[B_RAW + sl], kRawBytes);
            tma_load_3d(sm + Ly::RAW + sl * kRawBytes, map_of(w), &bars[B_RAW + sl], h * kD, row0(c0 + i), b);
            if (i + 1 < n) tma_prefetch_3d(map_of(w), h * kD, max(row0(c0 + i + 1), 0), b);
        };
        int issued_hi = -1, consumed_hi = -1;  // thread 0: last load issued / read
        if (pt == 0) {
            for (int l = 0; l < NSL && l < nload; ++l) issue(l);
            issued_hi = min(NSL, nload) - 1;
        }
        // the head's conv taps, once: [tensor][j][cg] so that a token row's 16 threads read 16
        // consecutive float4
        for (int e = pt; e < NT * 128; e += 128) {
            const int w = e >> 7, ch = e & 127;
            convs[w * 128 + (ch & 7) * 16 + (ch >> 3)] =
                __ldg(reinterpret_cast<const float4 *>(conv_of(w)) + static_cast<size_t>(h) * kD + ch);
        }
        named_sync(NB_PREP, 128);
        bool ok = true;
        for (int i = 0; ok && i < n; ++i) {
            const int c = c0 + i, s = i & 1;
            uint8_t *kq = sm + Ly::KQ + s * 32768;
            const bool ragged = (c + 1) * kC > p.T;
            if (pt == 0) FTRACE(i, 8);
            if (i >= 2) ok = mbar_wait_ol(&bars[B_FREE + s], ((i >> 1) - 1) & 1, ab, p.status, lim);
#pragma unroll 1
            for (int w = 0; w < NT; ++w) {
                // destination: output pass k -> KQ rows 0-63, q -> KQ rows 64+, v -> V tile;
                // transfer pass k -> KQ rows 0-63, v -> KQ rows 64+
                const bool is_v = w == NT - 1;
                uint8_t *dst = kq;
                int drows = 128, doff = (w == 1) ? 64 : 0;
                if (kOut && is_v) {
                    dst = sm + Lay<true>::V;
                    drows = 64;
                    doff = 0;
                    if (i >= 1) ok = ok && mbar_wait_ol(&bars[B_VFREE], (i - 1) & 1, ab, p.status, lim);
                }
                const int l = i * NT + w, sl = l % NSL;
                ok = ok && mbar_wait_ol(&bars[B_RAW + sl], (l / NSL) & 1, ab, p.status, lim);
                ok = group_all(NB_PREP, 128, ok);
                if (!ok) break;
                if (pt == 0) FTRACE(i, 9 + 2 * w);
                consumed_hi = l;
                const uint8_t *tile = sm + Ly::RAW + sl * kRawBytes + cg * 16;
                float4 wt[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) wt[j] = convs[w * 128 + j * 16 + cg];
                // box row of window row k (k = 0 .. 66; the reverse scan reads its box bottom-up)
                const uint8_t *rp = tile + (p.rev ? (kRawRows - 1 - rbeg) * 256 : rbeg * 256);
                const int rstep = p.rev ? -256 : 256;
                // u_t = w0 x_(t-3) + w1 x_(t-2) + w2 x_(t-1) + w3 x_t: each raw row x_t completes u_t
                // and feeds the partial sums p0, p1, p2 of u_(t+1), u_(t+2), u_(t+3)
                float p0[8], p1[8], p2[8], ss[8], x[8];
                load8<InT>(rp, x);
#pragma unroll
                for (int j = 0; j < 8; ++j) p0[j] = wt[j].x * x[j];
                load8<InT>(rp + rstep, x);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    p0[j] = fmaf(wt[j].y, x[j], p0[j]);
                    p1[j] = wt[j].x * x[j];
                }
                load8<InT>(rp + 2 * rstep, x);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    p0[j] = fmaf(wt[j].z, x[j], p0[j]);
                    p1[j] = fmaf(wt[j].y, x[j], p1[j]);
                    p2[j] = wt[j].x * x[j];
                }
#pragma unroll
                for (int r = 0; r < 8; ++r) {
                    load8<InT>(rp + (r + 3) * rstep, x);
                    float u[8];
                    ss[r] = 0.0f;
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        u[j] = silu_tc(fmaf(wt[j].w, x[j], p0[j]));
                        p0[j] = fmaf(wt[j].z, x[j], p1[j]);
                        p1[j] = fmaf(wt[j].y, x[j], p2[j]);
                        p2[j] = wt[j].x * x[j];
                        ss[r] = fmaf(u[j], u[j], ss[r]);
                    }
                    if (ragged && c * kC + rbeg + r >= p.T) {
#pragma unroll
                        for (int j = 0; j < 8; ++j) u[j] = 0.0f;
                    }
                    put8h(dst, drows, doff + rbeg + r, cg, u);
                }
                if (!is_v) {
                    // |x'|^2 of the run's eight tokens over the 16 threads of each token row, as eight
                    // independent chains; then 1/|k'| or 1/(sqrt(d_k) |q'|) (padding tokens: their
                    // zero rows make the factor irrelevant)
#pragma unroll
                    for (int off = 8; off > 0; off >>= 1)
#pragma unroll
                        for (int r = 0; r < 8; ++r) ss[r] += __shfl_xor_sync(0xffffffffu, ss[r], off);
                    if (cg == 0) {
                        const float sc = (kOut && w == 1) ? p.q_scale : 1.0f;
                        float *dn = invn + s * 128 + (w == 1 ? 64 : 0) + rbeg;
#pragma unroll
                        for (int r = 0; r < 8; ++r) dn[r] = rsqrtf(ss[r] + p.l2_eps) * sc;
                    }
                }
                named_sync(NB_PREP, 128);  // every read of this raw box is done
                if (pt == 0) FTRACE(i, 10 + 2 * w);
                if (pt == 0 && l + NSL < nload) {
                    issue(l + NSL);
                    issued_hi = l + NSL;
                }
                if (w == 1 || (kOut && is_v)) {
                    fence_proxy_async();  // the tiles are read by the tensor cores next
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars[is_v && kOut ? B_PREPV : B_PREP + s]);
                }
            }
            if (!ok) break;
            if (pt == 0) FTRACE(i, 15);
        }
        if (pt == 0) {  // raw boxes still in flight land before shared memory goes away
            for (int l = consumed_hi + 1; l <= issued_hi; ++l)
                mbar_wait_drain(&bars[B_RAW + l % NSL], (l / NSL) & 1, lim);
        }
    } else if (warp < W_CH) {
        // ================================================================ gates, L, Aqk, Qt, T
        // Per block j: the gates (into the slot of block j - 2, free once the state warps have
        // finished that block's W^T tile and Kt), then from the block's Gram the rows of L (lanes
        // 0-63: K'K'^T) and of Aqk (lanes 64-127: Q'K'^T) and Qt, then T = (I + L)^-1 and the two
        // scaled T tiles of the slot (free once block j - 2's W^T and U^T are done).
        const int ut = tid - 32 * W_UT;
        const int q4 = warp & 3;
        const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
        const float eA = __expf(p.A_log[h]), dtb = p.dt_bias[h];
        bool ok = true;
        for (int j = 0; ok && j < n; ++j) {
            const int c = c0 + j, s = j & 1;
            float *Gs = gate + s * 256, *Bs = Gs + 64, *Ec = Gs + 128, *Bw = Gs + 192;
            const float *ik = invn + s * 128, *iq = ik + 64;  // 1/|k'|, 1/(sqrt(d_k) |q'|) of the tokens
            uint8_t *kq = sm + Ly::KQ + s * 32768;
            uint8_t *Tt = sm + Ly::T + s * 8192, *TWt = sm + Ly::TW + s * 8192;
            if (ut == 0) FTRACE(j, 16);
            // ---- gates: log alpha = -exp(A_log) softplus(g + dt_bias), beta = sigmoid(b), G = inclusive
            //      cumulative sum of log alpha over the block (padding rows: 0, 0), and the column factors
            //      e^(G_m - G_j) of the split decay (m the last row of j's 16-row group)
            ok = group_all(NB_UT, 128, j < 2 || mbar_wait_ol(&bars[B_UTD + s], ((j >> 1) - 1) & 1, ab, p.status, lim));
            if (!ok) break;
            {
                float cs = 0.0f, be = 0.0f;
                if (ut < 64) {
                    const int t = c * kC + ut;
                    float la = 0.0f;
                    if (t < p.T) {
                        const size_t gi = (static_cast<size_t>(b) * p.T + (p.rev ? p.T - 1 - t : t)) * p.H + h;
                        if (p.debug && gi >= static_cast<size_t>(p.B) * p.T * p.H) {
                            atomicCAS(p.status, kStatusOk, kStatusCheck);
                        } else {
                            const float xg = p.g[gi] + dtb;
                            const float sp = xg > 20.0f ? xg : __logf(1.0f + __expf(xg));
                            la = -eA * sp;
                            be = __fdividef(1.0f, 1.0f + __expf(-p.bg[gi]));
                        }
                    }
                    cs = la;
#pragma unroll
                    for (int off = 1; off < 32; off <<= 1) {
                        const float v = __shfl_up_sync(0xffffffffu, cs, off);
                        if (lane >= off) cs += v;
                    }
                    if (lane == 31) wtot[ut >> 5] = cs;
                }
                named_sync(NB_UT, 128);
                if (ut < 64) {
                    Gs[ut] = cs + (ut >= 32 ? wtot[0] : 0.0f);
                    Bs[ut] = be;
                }
                named_sync(NB_UT, 128);
                if (ut < 64) Ec[ut] = __expf(fminf(Gs[ut | 15] - Gs[ut], 0.0f));
                named_sync(NB_UT, 128);
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[B_GATE + s]);
            }
            if (ut == 0) FTRACE(j, 17);
            // ---- L and Aqk rows; Qt
            ok = group_all(NB_UT, 128,
                           mbar_wait_ol(&bars[B_PREP + s], (j >> 1) & 1, ab, p.status, lim) &&
                               mbar_wait_ol(&bars[B_GRAM], j & 1, ab, p.status, lim) &&
                               (j < 2 || mbar_wait_ol(&bars[B_WT + s], ((j >> 1) - 1) & 1, ab, p.status, lim)));
            if (!ok) break;
            if (ut == 0) FTRACE(j, 18);
            tc_fence_after();
            {
                const int r = (q4 & 1) * 32 + lane;  // row within the block
                const bool lrow = q4 < 2;
                if (lrow || kOut) {
                    // L_rj = beta_r e^(G_r - G_j) k_r.k_j (j < r);  Aqk_rj = e^(G_r - G_j) q_r.k_j / sqrt(d_k)
                    // (j <= r); below r's 16-row group the decay splits as e^(G_r - G_m) e^(G_m - G_j)
                    const float Gr = Gs[r];
                    const float br = lrow ? Bs[r] * ik[r] : iq[r];
                    uint8_t *dstt = lrow ? Tt : (sm + (kOut ? Lay<true>::AQK : 0) + s * 8192);
                    const int rg16 = r >> 4;
                    const int lim_j = lrow ? r : r + 1;  // columns j < lim_j are kept
#pragma unroll 1
                    for (int g = 0; g < 4; ++g) {
                        float a[16], l[16];
                        tmem_ld16(tmem + lane_base + TM::GA + g * 16, a);
                        if (g < rg16) {
                            const float fr = br * __expf(fminf(Gr - Gs[16 * g + 15], 0.0f));
#pragma unroll
                            for (int e = 0; e < 16; ++e) l[e] = fr * Ec[16 * g + e] * ik[16 * g + e] * a[e];
                        } else {
#pragma unroll
                            for (int e = 0; e < 16; ++e) {
                                const int jj = 16 * g + e;
                                l[e] = (jj < lim_j) ? br * __expf(fminf(Gr - Gs[jj], 0.0f)) * ik[jj] * a[e] : 0.0f;
                            }
                            if (lrow && g == rg16) {
                                float *dd = ldiag + rg16 * 256 + (r & 15) * 16;
#pragma unroll
                                for (int e = 0; e < 16; e += 4)
                                    *reinterpret_cast<float4 *>(dd + e) = make_float4(l[e], l[e + 1], l[e + 2], l[e + 3]);
                            }
                        }
                        put8h(dstt, 64, r, 2 * g, l);
                        put8h(dstt, 64, r, 2 * g + 1, l + 8);
                    }
                    if (kOut && !lrow) scale_row_chunks(kq, 128, 64 + r, 0, 16, __expf(fminf(Gr, 0.0f)) * iq[r]);  // Qt
                }
                if (ut < 64) Bw[ut] = Bs[ut] * __expf(Gs[ut]) * ik[ut];
            }
            tc_fence_before();
            named_sync(NB_UT, 128);
            if (ut == 0) FTRACE(j, 19);
            // ---- T = (I + L)^-1, then T diag(beta e^G / |k'|) (TW tile) and T diag(beta) (in place)
            invert_unit_lower64(Tt, ldiag, ut);
            if (ut == 0) FTRACE(j, 20);
            {
                const int rr = ut >> 1, ch0 = (ut & 1) * 4;
#pragma unroll
                for (int ch = ch0; ch < ch0 + 4; ++ch) {
                    uint4 *pu = reinterpret_cast<uint4 *>(Tt + tile_off(64, rr, ch));
                    const uint4 u = *pu;
                    const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
                    uint32_t ow[4], ou[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 xx = unpack_half2(w4[e]);
                        const int jj = ch * 8 + 2 * e;
                        ow[e] = pack_half2(xx.x * Bw[jj], xx.y * Bw[jj + 1]);
                        ou[e] = pack_half2(xx.x * Bs[jj], xx.y * Bs[jj + 1]);
                    }
                    *reinterpret_cast<uint4 *>(TWt + tile_off(64, rr, ch)) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
                    *pu = make_uint4(ou[0], ou[1], ou[2], ou[3]);
                }
            }
            fence_proxy_async();
            named_sync(NB_UT, 128);
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_TREADY + s]);
            if (ut == 0) FTRACE(j, 21);
        }
    } else if (warp < W_X || !kOut) {
        // ================================================================ state step
        // warps 9-12: the state S (lanes = d_v), and each block's W^T tile and Kt (lanes = d_k);
        // transfer pass warps 13-16: the transfer P (lanes = d_k)
        const bool isP = !kOut && warp >= W_X;
        const int q4 = warp & 3;
        const int row = q4 * 32 + lane;
        const uint32_t lb = static_cast<uint32_t>(q4 * 32) << 16;
        const uint32_t tN = tmem + lb + (isP ? Tm<false>::NP : TM::N);
        const uint32_t tU = tmem + lb + (isP ? Tm<false>::UDP : TM::UD);
        const uint32_t tE = tmem + lb + (isP ? Tm<false>::E16P : TM::E16);
        uint8_t *n16s = kOut ? nullptr : sm + (isP ? Lay<false>::N16P : Lay<false>::N16S);
        // columns 32 ch .. 32 ch + 31 of the fp16 state copy the next MMAs read: TMEM (output pass,
        // two fp16 per column) or row `row` of a K-major tile (transfer pass)
        auto put_n16 = [&](const float (&v)[32], int ch) {
            if constexpr (kOut) {
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) pk[e] = pack_half2(v[2 * e], v[2 * e + 1]);
                tmem_st16(tmem + lb + Tm<true>::N16 + ch * 16, pk);
            } else {
#pragma unroll
                for (int q = 0; q < 4; ++q) put8h(n16s, 128, row, ch * 4 + q, v + 8 * q);
            }
        };
        // initial (negated) state: row `row` of S_start, or -I for the transfer matrix; its fp16 copy,
        // then the state decayed by the first block's decay
        bool ok = true;
        {
            const float *src = nullptr;
            if (!isP) {
                if (seg == 0) {
                    src = p.s0 ? p.s0 + (static_cast<size_t>(bh) * kD + row) * kD : nullptr;
                } else if (kOut) {
                    pdl_wait();  // the combine's segment start states are complete
                    src = p.SS + ((static_cast<size_t>(bh) * p.NS + seg) * kD + row) * kD;
                }
            }
            ok = __all_sync(0xffffffffu, mbar_wait_ol(&bars[B_GATE], 0, ab, p.status, lim));
            const float gC = ok ? __expf(fminf(gate[kC - 1], 0.0f)) : 0.0f;
#pragma unroll 1
            for (int ch = 0; ch < 4; ++ch) {
                float v[32];
#pragma unroll
                for (int e = 0; e < 32; e += 4) {
                    float4 xv = src ? *reinterpret_cast<const float4 *>(src + ch * 32 + e) : make_float4(0.f, 0.f, 0.f, 0.f);
                    if (isP) {
                        xv.x = (ch * 32 + e == row) ? 1.0f : 0.0f;
                        xv.y = (ch * 32 + e + 1 == row) ? 1.0f : 0.0f;
                        xv.z = (ch * 32 + e + 2 == row) ? 1.0f : 0.0f;
                        xv.w = (ch * 32 + e + 3 == row) ? 1.0f : 0.0f;
                    }
                    v[e] = -xv.x; v[e + 1] = -xv.y; v[e + 2] = -xv.z; v[e + 3] = -xv.w;
                }
                put_n16(v, ch);
#pragma unroll
                for (int e = 0; e < 32; ++e) v[e] *= gC;
                tmem_st32(tN + ch * 32, v);
            }
            tmem_st_wait();
            if (!kOut) fence_proxy_async();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_N16]);
        }
        for (int i = 0; ok && i < n; ++i) {
            const int s = i & 1;
            if (!isP) {
                // ---- block i's W^T (lanes = d_k) into its slot's tile, and Kt = diag(e^(G_C - G) / |k'|) K'
                ok = __all_sync(0xffffffffu, mbar_wait_ol(&bars[B_WT + s], (i >> 1) & 1, ab, p.status, lim) &&
                                                 mbar_wait_ol(&bars[B_PREP + s], (i >> 1) & 1, ab, p.status, lim) &&
                                                 mbar_wait_ol(&bars[B_GATE + s], (i >> 1) & 1, ab, p.status, lim));
                if (!ok) break;
                if (tid == 32 * W_CH) FTRACE(i, 24);
                tc_fence_after();
                {
                    float a[32], a2[32];
                    tmem_ld32x2(tmem + lb + TM::GB, tmem + lb + TM::GB + 32, a, a2);
                    uint8_t *wt = sm + Ly::WT + s * 16384;
#pragma unroll
                    for (int q = 0; q < 4; ++q) put8h(wt, 128, row, q, a + 8 * q);
#pragma unroll
                    for (int q = 0; q < 4; ++q) put8h(wt, 128, row, 4 + q, a2 + 8 * q);
                }
                {
                    const float *Gs = gate + s * 256, *ik = invn + s * 128;
                    const int r = row >> 1;
                    scale_row_chunks(sm + Ly::KQ + s * 32768, 128, r, (row & 1) * 8, 8,
                                     __expf(fminf(Gs[kC - 1] - Gs[r], 0.0f)) * ik[r]);
                }
                fence_proxy_async();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[B_UTD + s]);
            }
            // ---- Delta^T -> E16 = fp16(-Delta^T), written over the first half of its columns
            ok = __all_sync(0xffffffffu, mbar_wait_ol(&bars[B_DELTA], i & 1, ab, p.status, lim));
            if (!ok) break;
            if (tid == 32 * W_CH) FTRACE(i, 25);
            tc_fence_after();
            {
                float d0[32], d1[32];
                uint32_t pk[16];
                tmem_ld32x2(tU, tU + 32, d0, d1);
#pragma unroll
                for (int e = 0; e < 16; ++e) pk[e] = pack_half2(-d0[2 * e], -d0[2 * e + 1]);
                tmem_st16(tE, pk);
#pragma unroll
                for (int e = 0; e < 16; ++e) pk[e] = pack_half2(-d1[2 * e], -d1[2 * e + 1]);
                tmem_st16(tE + 16, pk);
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_E16]);
            if (tid == 32 * W_CH) FTRACE(i, 26);
            ok = __all_sync(0xffffffffu, mbar_wait_ol(&bars[B_STATE], i & 1, ab, p.status, lim));
            if (!ok) break;
            if (tid == 32 * W_CH) FTRACE(i, 27);
            if (i + 1 < n) {
                // one read of the state: its fp16 copy for block i + 1's products, and the state
                // decayed by block i + 1's total decay for its update
                const int s1 = (i + 1) & 1;
                ok = __all_sync(0xffffffffu, mbar_wait_ol(&bars[B_GATE + s1], ((i + 1) >> 1) & 1, ab, p.status, lim));
                if (!ok) break;
                const float gC = __expf(fminf(gate[s1 * 256 + kC - 1], 0.0f));
                tc_fence_after();
#pragma unroll 1
                for (int hf = 0; hf < 2; ++hf) {
                    float a[32], a2[32];
                    tmem_ld32x2(tN + hf * 64, tN + hf * 64 + 32, a, a2);
                    put_n16(a, 2 * hf);
                    put_n16(a2, 2 * hf + 1);
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        a[e] *= gC;
                        a2[e] *= gC;
                    }
                    tmem_st32(tN + hf * 64, a);
                    tmem_st32(tN + hf * 64 + 32, a2);
                }
                tmem_st_wait();
                if (!kOut) fence_proxy_async();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[B_N16]);
                if (tid == 32 * W_CH) FTRACE(i, 28);
            } else {
                // end of the segment: S_loc / P (transfer pass), or the final state
                float *dst = nullptr;
                if (!kOut) dst = p.SP + ((static_cast<size_t>(bh) * p.NS + seg) * 2 + (isP ? 1 : 0)) * kD * kD;
                else if (p.s_end && seg == p.NS - 1) dst = p.s_end + static_cast<size_t>(bh) * kD * kD;
                if (dst) {
                    tc_fence_after();
                    float *d = dst + static_cast<size_t>(row) * kD;
#pragma unroll 1
                    for (int ch = 0; ch < 4; ++ch) {
                        float v[32];
                        tmem_ld32(tN + ch * 32, v);
#pragma unroll
                        for (int e = 0; e < 32; e += 4)
                            *reinterpret_cast<float4 *>(d + ch * 32 + e) = make_float4(-v[e], -v[e + 1], -v[e + 2], -v[e + 3]);
                    }
                }
            }
        }
    } else {
        // ================================================================ output step (output pass)
        // y = o / sqrt(mean(o^2) + eps) * w * SiLU(z), o = -(the O^T accumulator), lanes = d_v
        const int et = tid - 32 * W_X;
        const int q4 = warp & 3;
        const int row = q4 * 32 + lane;  // d_v channel (TMEM lane)
        const uint32_t lb = static_cast<uint32_t>(q4 * 32) << 16;
        uint8_t *zt = sm + Lay<true>::Z;
        const bool zhalf = std::is_same<InT, __half>::value;
        auto zrow0 = [&](int c) { return p.rev ? p.T - kC * (c + 1) : kC * c; };  // first row of block c's box
        int zpend = -1;  // thread 0: block whose z box is in flight and not yet consumed
        if (et == 0) {
            mbar_arrive_expect_tx(&bars[B_Z], kC * 256);
            tma_load_3d(zt, &tmz, &bars[B_Z], h * kD, zrow0(c0), b);
            if (n > 1) tma_prefetch_3d(&tmz, h * kD, max(zrow0(c0 + 1), 0), b);
            zpend = 0;
        }
        const float nwv = -nw[row];  // the O^T accumulator holds -o
        // row t of the z / y box (the reverse scan's box runs backwards)
        uint8_t *zrow = zt + (p.rev ? (kC - 1) * 256 : 0) + row * 2;
        const int zstep = p.rev ? -256 : 256;
        bool ok = true;
        for (int i = 0; ok && i < n; ++i) {
            const int c = c0 + i, s = i & 1;
            const uint32_t tO = tmem + lb + Tm<true>::O + s * 64;
            ok = group_all(NB_X, 128, mbar_wait_ol(&bars[B_OFULL + s], (i >> 1) & 1, ab, p.status, lim));
            if (!ok) break;
            if (et == 0) FTRACE(i, 29);
            tc_fence_after();
            // sum over the 128 channels of o^2 per token: reduce-scatter across the warp's lanes, 32
            // tokens at a time (lane l ends with token 32 hf + l), then across the four warps
#pragma unroll 1
            for (int hf = 0; hf < 2; ++hf) {
                float x[32];
                tmem_ld32(tO + hf * 32, x);
#pragma unroll
                for (int e = 0; e < 32; ++e) x[e] *= x[e];
#pragma unroll
                for (int lvl = 0; lvl < 5; ++lvl) {
                    const int half = 16 >> lvl;  // current length 2 * half
                    const bool up = (lane & half) != 0;
#pragma unroll
                    for (int jj = 0; jj < 16; ++jj) {
                        if (jj < half) {
                            const float send = up ? x[jj] : x[jj + half];
                            const float keep = up ? x[jj + half] : x[jj];
                            x[jj] = keep + __shfl_xor_sync(0xffffffffu, send, half);
                        }
                    }
                }
                red[(hf * 32 + lane) * 4 + q4] = x[0];
            }
            named_sync(NB_X, 128);
            if (et < 64) {
                const float4 r4 = *reinterpret_cast<const float4 *>(red + et * 4);
                rns[et] = rsqrtf((r4.x + r4.y + r4.z + r4.w) * (1.0f / 128.0f) + p.eps);
            }
            ok = group_all(NB_X, 128, mbar_wait_ol(&bars[B_Z], i & 1, ab, p.status, lim));  // (also publishes rns)
            if (!ok) break;
            if (et == 0) {
                FTRACE(i, 30);
                zpend = -1;
            }
            bool bad = false;
            // padding rows have o = 0 and z = 0, so y = 0 there; only fp32 outputs, stored directly,
            // need the live-row test
#pragma unroll 1
            for (int ch = 0; ch < 4; ++ch) {  // 16 tokens at a time
                float o[16];
                tmem_ld16(tO + ch * 16, o);
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int t = ch * 16 + e;
                    uint8_t *zp = zrow + t * zstep;
                    const float yv = o[e] * (rns[t] * nwv) * silu_tc(load1(zp, zhalf));
                    bad |= !isfinite(yv);
                    if (p.out_kind == 1) {
                        const int tt = c * kC + t;
                        if (tt < p.T) {
                            const int xr = p.rev ? p.T - 1 - tt : tt;
                            static_cast<float *>(p.y)[((static_cast<size_t>(b) * p.T + xr) * p.H + h) * kD + row] = yv;
                        }
                    } else if (p.out_kind == 0) {
                        *reinterpret_cast<__nv_bfloat16 *>(zp) = __float2bfloat16_rn(yv);
                    } else {
                        *reinterpret_cast<__half *>(zp) = __float2half_rn(yv);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_OFREE + s]);
            if (p.debug && bad) atomicCAS(p.status, kStatusOk, kStatusCheck);
            if (p.out_kind != 1) fence_proxy_async();
            named_sync(NB_X, 128);  // every read of the z box (and write of the y box) is done
            if (et == 0) {
                if (p.out_kind != 1) {
                    const int y0 = zrow0(c);
                    if (y0 >= 0) {
                        tma_store_3d(&tmy, zt, h * kD, y0, b);
                    } else {  // reverse scan, ragged last block: only its live rows, from token 0
                        tma_store_3d(&tmy_tail, zt + (-y0) * 256, h * kD, 0, b);
                    }
                    bulk_commit();
                    bulk_wait_read_all();
                }
                FTRACE(i, 31);
                if (i + 1 < n) {
                    mbar_arrive_expect_tx(&bars[B_Z], kC * 256);
                    tma_load_3d(zt, &tmz, &bars[B_Z], h * kD, zrow0(c + 1), b);
                    if (i + 2 < n) tma_prefetch_3d(&tmz, h * kD, max(zrow0(c + 2), 0), b);
                    zpend = i + 1;
                }
            }
        }
        if (et == 0) {
            if (zpend >= 0) mbar_wait_drain(&bars[B_Z], zpend & 1, lim);
            bulk_wait_all();
        }
    }

teardown:
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == W_MMA) tmem_dealloc(tmem, 512);
}

// ================================================================ combine
// S_start(1) = S_loc(0); S_start(j+1) = S_start(j) P_j + S_loc(j), sequential over j, in fp32 on
// CUDA cores.  Rows of S are independent: a CTA takes 8 rows (d_v) of one (b, h); thread
// (rr = tid / 32, cg = tid % 32) forms columns 4cg .. 4cg+3 of row rr.  P_j (128 x 128 fp32) is
// double-buffered in shared memory by cp.async, the copy of P_(j+1) in flight during step j.
constexpr int kCombRows = 8;
constexpr uint32_t kCombSmem = (2 * 128 * 128 + kCombRows * 128) * 4;

__global__ void __launch_bounds__(256) gdn_combine_kernel(const FusedParams p) {
    extern __shared__ __align__(16) float csm[];
    float *PT = csm;                 // [2][128][128]
    float *cur = csm + 2 * 128 * 128;  // [8][128]: rows of S_start(j)
    const int slice = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int bh = b * p.H + h;
    const int tid = threadIdx.x, rr = tid >> 5, cg = tid & 31;
    const int row = slice * kCombRows + rr;
    constexpr size_t kMat = 128 * 128;
    const float *SP = p.SP + static_cast<size_t>(bh) * p.NS * 2 * kMat;  // [NS][2][128][128]
    float *SS = p.SS + static_cast<size_t>(bh) * p.NS * kMat;
    pdl_launch_dependents();
    pdl_wait();  // the transfer pass's S_loc and P are complete
    auto load_p = [&](int j) {
        const float *src = SP + (static_cast<size_t>(j) * 2 + 1) * kMat;
        float *dst = PT + (j & 1) * kMat;
#pragma unroll 4
        for (int e = tid; e < 128 * 32; e += 256) cp_async16(dst + e * 4, src + e * 4);
        cp_async_commit();
    };
    if (p.NS > 2) load_p(1);
    float4 v = *reinterpret_cast<const float4 *>(SP + static_cast<size_t>(row) * 128 + cg * 4);  // S_loc(0)
    *reinterpret_cast<float4 *>(SS + (1 * kMat) + static_cast<size_t>(row) * 128 + cg * 4) = v;
    *reinterpret_cast<float4 *>(cur + rr * 128 + cg * 4) = v;
    for (int j = 1; j + 1 < p.NS; ++j) {
        const float4 sl = *reinterpret_cast<const float4 *>(SP + static_cast<size_t>(j) * 2 * kMat +
                                                            static_cast<size_t>(row) * 128 + cg * 4);
        if (j + 2 < p.NS) {
            load_p(j + 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();  // P_j and the current rows visible to all
        const float *P = PT + (j & 1) * kMat;
        const float *cr = cur + rr * 128;
        float a0 = sl.x, a1 = sl.y, a2 = sl.z, a3 = sl.w;
#pragma unroll 8
        for (int k = 0; k < 128; ++k) {
            const float sk = cr[k];
            const float4 pk = *reinterpret_cast<const float4 *>(P + k * 128 + cg * 4);
            a0 = fmaf(sk, pk.x, a0);
            a1 = fmaf(sk, pk.y, a1);
            a2 = fmaf(sk, pk.z, a2);
            a3 = fmaf(sk, pk.w, a3);
        }
        __syncthreads();  // every read of the current rows and of this P buffer is done
        const float4 o = make_float4(a0, a1, a2, a3);
        *reinterpret_cast<float4 *>(cur + rr * 128 + cg * 4) = o;
        *reinterpret_cast<float4 *>(SS + static_cast<size_t>(j + 1) * kMat + static_cast<size_t>(row) * 128 + cg * 4) = o;
    }
}

template <bool kOut, typename InT>
cudaError_t launch_pass(const FusedParams &p, const CUtensorMap *maps, cudaStream_t s, bool pdl) {
    static SmemOnce once;
    cudaError_t e = raise_smem_once(once, gdn_fused_kernel<kOut, InT>, static_cast<int>(smem_bytes<kOut>()));
    if (e != cudaSuccess) return e;
    dim3 grid(kOut ? p.NS : p.NS - 1, p.H, p.B);
    return launch_k(gdn_fused_kernel<kOut, InT>, grid, dim3(kThreads), smem_bytes<kOut>(), s, pdl, p, maps[0],
                    maps[1], maps[2], maps[3], maps[4], maps[5]);
}

}  // namespace

cudaError_t launch_fused_transfer(const FusedParams &p, InType in, const CUtensorMap *maps, cudaStream_t s,
                                  bool pdl) {
    return in == InType::F16 ? launch_pass<false, __half>(p, maps, s, pdl)
                             : launch_pass<false, __nv_bfloat16>(p, maps, s, pdl);
}

cudaError_t launch_fused_combine(const FusedParams &p, cudaStream_t s, bool pdl) {
    static SmemOnce once;
    cudaError_t e = raise_smem_once(once, gdn_combine_kernel, static_cast<int>(kCombSmem));
    if (e != cudaSuccess) return e;
    dim3 grid(128 / kCombRows, p.H, p.B);
    return launch_k(gdn_combine_kernel, grid, dim3(256), kCombSmem, s, pdl, p);
}

cudaError_t launch_fused_output(const FusedParams &p, InType in, const CUtensorMap *maps, cudaStream_t s, bool pdl) {
    return in == InType::F16 ? launch_pass<true, __half>(p, maps, s, pdl)
                             : launch_pass<true, __nv_bfloat16>(p, maps, s, pdl);
}

}  // namespace gdn

GDN_TRACE_EXPORT(fused)
