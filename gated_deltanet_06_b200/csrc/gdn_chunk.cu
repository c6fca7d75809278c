// gdn_chunk.cu -- the intra-block UT (WY) transform of the gated delta rule
// (reference [57] on the VMonarch page) on 5th-generation tensor cores.  One
// CTA handles one 128-token block of one (b, h):
//
//   A_kk = K K^T,  QK = Q K^T             tcgen05, fp16 x fp16 -> fp32 in TMEM
//   L_rj = beta_r exp(G_r - G_j) A_kk,rj  for j < r (decay-masked strict tril)
//   T    = (I + L)^-1                     blocked over 16x16 blocks (below)
//   W    = T diag(beta e^G) K,  U = T diag(beta) V      tcgen05
//   Kt   = diag(e^(G_last - G)) K,  Qt = diag(e^G) Q,
//   Aqk  = [i <= r] e^(G_r - G_i) QK_ri
//
// and stores W, U, Kt, Qt, Aqk (fp16) for the inter-block scan (TMA bulk
// stores for W, U, Qt; plain 16-byte stores for Kt and Aqk).  Only exponentials of non-positive differences of the cumulative
// log decay G are taken.
//
// T = (I + L)^-1 over the 8 x 8 grid of 16x16 blocks: the diagonal blocks
// D_i = (I + L_ii)^-1 by fp32 column solves (one thread per column, 16 rows);
// then three doubling levels, each joining pairs of inverted diagonal blocks
// of size n into inverses of size 2n by
//     [[A11, 0], [L21, A22]]^-1 = [[T11, 0], [-T22 L21 T11, T22]],
// as warp-level tensor-core products (mma.sync m16n8k16, fp16 operands
// fetched with ldmatrix from the swizzled tile, fp32 accumulation; the
// intermediate T22 L21 passes from accumulator to operand fragments in
// registers).  L and T live in one tile, each block overwritten in place
// once its last reader is done: T comes out directly in the K-major operand
// layout of W = T K~ and U = T V~.  Three dependent levels of two products
// each replace a 128-step serial solve.
//
// Two warp groups work side by side.  Warps 0-3 evaluate the gates, build L,
// invert I + L, then build Aqk and store it straight to global memory.  Warps
// 4-7 write Kt straight from the K tile to global memory while scaling the
// tile in place into K~ = diag(beta e^G) K, build Qt and store it, load the V
// tile and scale it into V~ = diag(beta) V, so that T enters both products
// unscaled.  The decay factors of L and Aqk
// below the diagonal 32x32 blocks are split as e^(G_r - G_m) e^(G_m - G_j) (m
// the last row of j's 32-row group, both exponents <= 0): one exponential per
// row and per column instead of one per entry.
//
// Footprint: about 108 KB of shared memory and 256 TMEM columns, so that two
// CTAs share an SM.  Shared memory is reused through the block's life: the K
// tile becomes K~; the Q tile becomes Qt, then V~, then the staging area of U;
// the L tile becomes T, then the staging area of W.
#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

// Shared-memory map (offsets from a 1024-byte aligned base).
constexpr uint32_t OFF_K = 0;           // 128x128 fp16 panel tile: K -> K~
constexpr uint32_t OFF_QV = 32768;      // 128x128 fp16: Q -> Qt -> V~ -> U staging
constexpr uint32_t OFF_LT = 65536;      // 128x128 fp16: L -> T (K-major A operand) -> W staging
constexpr uint32_t OFF_LDIAG = 98304;   // fp32 [8][16][16]: the diagonal 16x16 blocks of L
constexpr uint32_t OFF_G = OFF_LDIAG + 8192;    // fp32 [128]
constexpr uint32_t OFF_BETA = OFF_G + 512;      // fp32 [128]
constexpr uint32_t OFF_WT = OFF_BETA + 512;     // fp32 [4]: per-warp totals of the gate scan
constexpr uint32_t OFF_EC = OFF_WT + 16;        // fp32 [128]: e^(G_m - G_j), m = last row of j's 32-row group
constexpr uint32_t OFF_BAR = OFF_EC + 512;      // 3 mbarriers, tmem slot, abort flag
constexpr uint32_t SMEM_USED = OFF_BAR + 32;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // + alignment slack
static_assert(OFF_LT % 1024 == 0 && OFF_QV % 1024 == 0, "swizzle atoms need 1 KB alignment");
static_assert(SMEM_BYTES * 2 <= 227 * 1024, "two CTAs per SM");

constexpr uint32_t TM_AKK = 0, TM_QK = 128, TM_U = 128, TM_W = 0;  // 256 columns

// named barrier for one warp group (128 threads): 1 = warps 0-3, 2 = warps 4-7
__device__ __forceinline__ void group_sync(int id) { asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory"); }

__device__ __forceinline__ void put8(uint8_t *tile, int rows, int r, int chunk16, const float *v) {
    uint4 u;
    u.x = pack_half2(v[0], v[1]);
    u.y = pack_half2(v[2], v[3]);
    u.z = pack_half2(v[4], v[5]);
    u.w = pack_half2(v[6], v[7]);
    *reinterpret_cast<uint4 *>(tile + tile_off(rows, r, chunk16)) = u;
}

// Row r of a 128x128 fp16 panel tile, scaled by s in place.
__device__ __forceinline__ void scale_row(uint8_t *tile, int r, float s) {
#pragma unroll 4
    for (int c = 0; c < 16; ++c) {
        uint4 *pu = reinterpret_cast<uint4 *>(tile + tile_off(128, r, c));
        const uint4 u = *pu;
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 x = unpack_half2(w[e]);
            o[e] = pack_half2(x.x * s, x.y * s);
        }
        *pu = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// ------------------------------------------------ warp-level tensor-core products
// ldmatrix of four 8x8 fp16 matrices (the A operand of m16n8k16) / two transposed ones (B).
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
// d += a (16x16, row-major fragment) * b (16x8, column fragment), fp16 in, fp32 accumulate.
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

__global__ void __launch_bounds__(256, 2)
    gdn_chunk_kernel(const ChunkParams p, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmU,
                     const __grid_constant__ CUtensorMap tmQt, const __grid_constant__ CUtensorMap tmAqk,
                     const __grid_constant__ CUtensorMap tmAqkH, const __grid_constant__ CUtensorMap tmT) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    float *sG = reinterpret_cast<float *>(sm + OFF_G);
    float *sBeta = reinterpret_cast<float *>(sm + OFF_BETA);
    float *sEc = reinterpret_cast<float *>(sm + OFF_EC);
    uint64_t *bar_load = reinterpret_cast<uint64_t *>(sm + OFF_BAR);  // K and Q tiles
    uint64_t *bar_mma = bar_load + 1;
    uint64_t *bar_v = bar_load + 2;   // V tile
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_load + 3);
    AbortState *ab = reinterpret_cast<AbortState *>(tmem_slot + 1);

    const int blk = blockIdx.x, bh = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool groupL = tid < 128;  // warps 0-3: gates, L, T, Aqk;  warps 4-7: Kt, K~, Qt, V~
    const int r = tid & 127;        // TMEM lane / row (or column of T) owned by this thread
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const size_t row0 = static_cast<size_t>(bh) * p.Tp + static_cast<size_t>(blk) * kBlk;
    const int y0 = static_cast<int>(row0);
    // debug: the block's rows inside the [BH][Tp] gate and tile arrays, and its tokens inside T
    // rounded up to whole blocks (the gates of token t < T are read at [B][T][H])
    if (!debug_in_bounds(p.debug, row0, kBlk, static_cast<size_t>(p.BH) * p.Tp, p.status) ||
        !debug_in_bounds(p.debug, static_cast<size_t>(blk) * kBlk, kBlk, static_cast<size_t>(p.NB) * kBlk, p.status))
        return;

    if (tid == 0) {
        mbar_init(bar_load, 1);
        mbar_init(bar_mma, 1);
        mbar_init(bar_v, 1);
        ab->flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 256);
        tmem_relinquish();
    }
    // asynchronous work in flight, for the drain at teardown: tensor-core commits on bar_mma
    // (thread 0) and the V load on bar_v (thread 128)
    int mma_commits = 0;
    bool v_issued = false;
    pdl_launch_dependents();
    __syncthreads();  // barrier init visible before the TMA below uses it
    pdl_wait();       // the prep kernel's q^, k^, v^ are complete
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
        const size_t gi = t < p.T ? (static_cast<size_t>(bb) * p.T + (p.rev ? p.T - 1 - t : t)) * p.H + hh : 0;
        if (t < p.T && debug_in_bounds(p.debug, gi, 1, static_cast<size_t>(p.BH) * p.T, p.status)) {
            const float xg = p.g[gi] + p.dt_bias[hh];
            const float sp = xg > 20.0f ? xg : __logf(1.0f + __expf(xg));
            la = -__expf(p.A_log[hh]) * sp;
            be = __fdividef(1.0f, 1.0f + __expf(-p.bg[gi]));
        }
        float cs = la;
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
    if (tid == 0) GDN_TRACE_AT(0);
    mbar_wait(bar_load, 0, ab, p.status, p.wait_limit_ns);
    if (tid == 0) GDN_TRACE_AT(1);
    __syncthreads();
    if (ab->flag) goto teardown;

    // ---- A_kk = K K^T and Q K^T (M = N = K = 128; both operands K-major); bar_mma phase 0
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
        ++mma_commits;
    }
    mbar_wait(bar_mma, 0, ab, p.status, p.wait_limit_ns);
    __syncthreads();
    if (ab->flag) goto teardown;
    tc_fence_after();

    if (groupL) {
        // ---- L row r (fp16, into the L tile), and its diagonal 16x16 block in fp32.  Warp w owns
        //      rows 32w .. 32w+31: column group c < w lies wholly below the diagonal (split decay,
        //      no exponential per entry), c == w holds the diagonal, c > w is zero and never read.
        const float Gr = sG[r], br = sBeta[r];
        float *Ldg = reinterpret_cast<float *>(sm + OFF_LDIAG);
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
                const bool hi = (r & 16) != 0;  // which 16-column half holds this row's diagonal block
                float *dst = Ldg + (r >> 4) * 256 + (r & 15) * 16;
#pragma unroll
                for (int e = 0; e < 16; e += 4)
                    *reinterpret_cast<float4 *>(dst + e) =
                        make_float4(hi ? l[16 + e] : l[e], hi ? l[17 + e] : l[e + 1], hi ? l[18 + e] : l[e + 2],
                                    hi ? l[19 + e] : l[e + 3]);
            }
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) put8(sm + OFF_LT, 128, r, c * 4 + q4, &l[q4 * 8]);
        }
        group_sync(1);
        if (tid == 0) GDN_TRACE_AT(2);

        // ---- diagonal blocks D_b = (I + L_bb)^-1: thread r solves column r % 16 of block r / 16
        //      (fp32) and writes it over L_bb, then zeros row r right of its diagonal block
        {
            const int b = r >> 4, c = r & 15;
            const float *Lb = Ldg + b * 256;
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
            uint8_t *Tt = sm + OFF_LT;
#pragma unroll
            for (int rr = 0; rr < 16; ++rr)
                *reinterpret_cast<__half *>(Tt + tile_elem_off(128, 16 * b + rr, r)) = __float2half_rn(x[rr]);
            for (int ch = 2 * b + 2; ch < 16; ++ch)
                *reinterpret_cast<uint4 *>(Tt + tile_off(128, r, ch)) = make_uint4(0, 0, 0, 0);
        }
        group_sync(1);
        if (tid == 0) GDN_TRACE_AT(3);

        // ---- T by recursive doubling over the diagonal blocks: with the 16x16 inverses D_b on the
        //      diagonal and L below it, level s (s = 1, 2, 3) joins pairs of 2^(s-1) blocks into
        //      inverses of 2^s blocks: for [[A11, 0], [L21, A22]], T21 = -T22 L21 T11.  Z = T22 L21
        //      accumulates in registers (fp32), becomes the A operand of Z T11 in fp16, and -Z T11 is
        //      written over L21.  Warp w computes block row(s) of its own output; a barrier separates
        //      the last read of a level's L21 from the first write over it.
        const uint32_t tT = sbase + OFF_LT;
        uint8_t *Tt = sm + OFF_LT;
        const int g = lane >> 2, t4 = lane & 3;
        const int lm = lane >> 3, lr = lane & 7;
        const int arow = (lm & 1) * 8 + lr, achk = lm >> 1;  // ldmatrix row / 16-byte chunk of this lane
        // A fragment of block (R, K); B fragments (two 8-column halves) of block (K, J)
        auto lda = [&](int R, int K, uint32_t (&a)[4]) { ldsm_x4(tT + tile_off(128, 16 * R + arow, 2 * K + achk), a); };
        auto ldb = [&](int K, int J, int hf, uint32_t (&b)[2]) {
            ldsm_x2_trans(tT + tile_off(128, 16 * K + arow, 2 * J + hf), b);
        };
        // C fragments (two 8-column halves of a 16x16 block) -> the A fragment of that block, fp16
        auto c2a = [&](const float (&c0)[4], const float (&c1)[4], uint32_t (&a)[4]) {
            a[0] = pack_half2(c0[0], c0[1]);
            a[1] = pack_half2(c0[2], c0[3]);
            a[2] = pack_half2(c1[0], c1[1]);
            a[3] = pack_half2(c1[2], c1[3]);
        };
        auto put_neg = [&](int R, int J, const float (&c0)[4], const float (&c1)[4]) {
            const int col = 16 * J + 2 * t4;
            *reinterpret_cast<uint32_t *>(Tt + tile_elem_off(128, 16 * R + g, col)) = pack_half2(-c0[0], -c0[1]);
            *reinterpret_cast<uint32_t *>(Tt + tile_elem_off(128, 16 * R + g + 8, col)) = pack_half2(-c0[2], -c0[3]);
            *reinterpret_cast<uint32_t *>(Tt + tile_elem_off(128, 16 * R + g, col + 8)) = pack_half2(-c1[0], -c1[1]);
            *reinterpret_cast<uint32_t *>(Tt + tile_elem_off(128, 16 * R + g + 8, col + 8)) = pack_half2(-c1[2], -c1[3]);
        };
        // level 1: pairs (2w, 2w+1), one per warp: T_{2w+1,2w} = -D_{2w+1} L_{2w+1,2w} D_{2w}
        {
            const int R = 2 * warp + 1, J = 2 * warp;
            uint32_t a[4], b[2];
            float z0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, z1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            lda(R, R, a);
            ldb(R, J, 0, b);
            mma16816(z0, a, b);
            ldb(R, J, 1, b);
            mma16816(z1, a, b);
            c2a(z0, z1, a);
            float y0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, y1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            ldb(J, J, 0, b);
            mma16816(y0, a, b);
            ldb(J, J, 1, b);
            mma16816(y1, a, b);
            __syncwarp();
            put_neg(R, J, y0, y1);
        }
        group_sync(1);
        if (tid == 0) GDN_TRACE_AT(20);
        // level 2: 64-blocks q = 0, 1 (blocks 4q .. 4q+3); warp w takes output block row R = 4q+2+i
        {
            const int q = warp >> 1, i = warp & 1;
            const int R = 4 * q + 2 + i, J0 = 4 * q;
            float z[2][2][4];
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int h = 0; h < 2; ++h) z[j][h][0] = z[j][h][1] = z[j][h][2] = z[j][h][3] = 0.0f;
            for (int K = 4 * q + 2; K <= R; ++K) {  // Z = T22 L21, row R
                uint32_t a[4];
                lda(R, K, a);
#pragma unroll
                for (int j = 0; j < 2; ++j)
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        uint32_t b[2];
                        ldb(K, J0 + j, h, b);
                        mma16816(z[j][h], a, b);
                    }
            }
            group_sync(1);  // every read of this level's L21 is done
            uint32_t za[2][4];
#pragma unroll
            for (int j = 0; j < 2; ++j) c2a(z[j][0], z[j][1], za[j]);
#pragma unroll
            for (int j = 0; j < 2; ++j) {  // Y = Z T11, row R: Y_j = sum_{k >= j} Z_k T11_kj
                float y0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, y1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
                for (int k = j; k < 2; ++k) {
                    uint32_t b[2];
                    ldb(J0 + k, J0 + j, 0, b);
                    mma16816(y0, za[k], b);
                    ldb(J0 + k, J0 + j, 1, b);
                    mma16816(y1, za[k], b);
                }
                put_neg(R, J0 + j, y0, y1);
            }
        }
        group_sync(1);
        if (tid == 0) GDN_TRACE_AT(21);
        // level 3: the 128-block; warp w takes output block row R = 4 + w
        {
            const int R = 4 + warp;
            float z[4][2][4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int h = 0; h < 2; ++h) z[j][h][0] = z[j][h][1] = z[j][h][2] = z[j][h][3] = 0.0f;
            for (int K = 4; K <= R; ++K) {  // Z = T22 L21, row R
                uint32_t a[4];
                lda(R, K, a);
#pragma unroll
                for (int j = 0; j < 4; ++j)
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        uint32_t b[2];
                        ldb(K, j, h, b);
                        mma16816(z[j][h], a, b);
                    }
            }
            group_sync(1);  // every read of L21 is done
            uint32_t za[4][4];
#pragma unroll
            for (int j = 0; j < 4; ++j) c2a(z[j][0], z[j][1], za[j]);
#pragma unroll
            for (int j = 0; j < 4; ++j) {  // Y = Z T11, row R
                float y0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, y1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
                for (int k = j; k < 4; ++k) {
                    uint32_t b[2];
                    ldb(k, j, 0, b);
                    mma16816(y0, za[k], b);
                    ldb(k, j, 1, b);
                    mma16816(y1, za[k], b);
                }
                put_neg(R, j, y0, y1);
            }
        }
        group_sync(1);
        if (tid == 0) GDN_TRACE_AT(22);
        fence_proxy_async();  // T is read by the tensor cores next
        if (p.save) {  // T kept for the backward: one bulk store of the finished tile
            group_sync(1);
            if (tid == 0) {
                tma_store_2d(&tmT, sm + OFF_LT, 0, y0);
                tma_store_2d(&tmT, sm + OFF_LT + 16384, 64, y0);
                bulk_commit();
            }
        }
        if (tid == 0) GDN_TRACE_AT(4);
        // ---- Aqk rows (the decay split as for the L rows), stored straight to global memory: a
        //      block's 128 rows are 32 contiguous KB.  Aqk is block lower triangular; its upper-right
        //      64x64 quadrant (zero) is never stored, the rest is, zeros above the diagonal included.
        {
            __half *arow_g = p.Aqk + (row0 + r) * 128;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                if (r < 64 && c >= 2 && !p.save) break;
                float a[32];
                if (c > warp) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) a[i] = 0.0f;
                } else {
                    tmem_ld32(tmem + lane_base + TM_QK + c * 32, a);
                    if (c < warp) {
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
                for (int q4 = 0; q4 < 4; ++q4) {
                    uint4 u;
                    u.x = pack_half2(a[8 * q4], a[8 * q4 + 1]);
                    u.y = pack_half2(a[8 * q4 + 2], a[8 * q4 + 3]);
                    u.z = pack_half2(a[8 * q4 + 4], a[8 * q4 + 5]);
                    u.w = pack_half2(a[8 * q4 + 6], a[8 * q4 + 7]);
                    *reinterpret_cast<uint4 *>(arow_g + c * 32 + q4 * 8) = u;
                }
            }
        }
    } else {
        // ---- Kt = e^(G_last - G) K straight to global memory, and the K tile scaled in place into
        //      K~ = diag(beta e^G) K (the A_kk product, K's last reader, is complete).  Each warp
        //      instruction covers two whole rows (lanes 0-15 and 16-31, one 16-byte piece each), so
        //      the global stores are 512 contiguous bytes; row scales come from their owner lanes.
        const float Gr = sG[r];
        const float fq = __expf(fminf(Gr, 0.0f));
        {
            const float fk = __expf(fminf(sG[kBlk - 1] - Gr, 0.0f)), sk = sBeta[r] * fq;
            const int wrow = (warp & 3) * 32, c = lane & 15;
#pragma unroll 4
            for (int m = 0; m < 16; ++m) {
                const int src = 2 * m + (lane >> 4);  // lane owning the row handled here
                const int row = wrow + src;
                const float fkr = __shfl_sync(0xffffffffu, fk, src), skr = __shfl_sync(0xffffffffu, sk, src);
                uint4 *pu = reinterpret_cast<uint4 *>(sm + OFF_K + tile_off(128, row, c));
                const uint4 u = *pu;
                const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
                uint32_t ot[4], os[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 x = unpack_half2(w4[e]);
                    ot[e] = pack_half2(x.x * fkr, x.y * fkr);
                    os[e] = pack_half2(x.x * skr, x.y * skr);
                }
                *reinterpret_cast<uint4 *>(p.Kt + (row0 + row) * 128 + c * 8) = make_uint4(ot[0], ot[1], ot[2], ot[3]);
                *pu = make_uint4(os[0], os[1], os[2], os[3]);
            }
        }
        if (tid == 128) GDN_TRACE_AT(10);
        // ---- Qt = e^G Q over the Q tile in place -> bulk store
        scale_row(sm + OFF_QV, r, fq);
        fence_proxy_async();
        group_sync(2);
        if (tid == 128) {
            tma_store_2d(&tmQt, sm + OFF_QV, 0, y0);
            tma_store_2d(&tmQt, sm + OFF_QV + 16384, 64, y0);
            bulk_commit();
            bulk_wait_read_all();
        }
        group_sync(2);
        if (tid == 128) GDN_TRACE_AT(11);
        if (tid == 128) {  // the Q area is free again: V goes into it
            mbar_arrive_expect_tx(bar_v, 32768u);
            tma_load_2d(sm + OFF_QV, &tmV, bar_v, 0, y0);
            tma_load_2d(sm + OFF_QV + 16384, &tmV, bar_v, 64, y0);
            v_issued = true;
        }
        if (tid == 128) GDN_TRACE_AT(12);
        // ---- V~ = diag(beta) V, row r
        if (mbar_wait(bar_v, 0, ab, p.status, p.wait_limit_ns)) scale_row(sm + OFF_QV, r, sBeta[r]);
        fence_proxy_async();
        if (tid == 128) GDN_TRACE_AT(13);
    }
    tc_fence_before();
    __syncthreads();  // T, V~ and K~ complete
    if (ab->flag) goto teardown;
    if (tid == 0) GDN_TRACE_AT(5);

    // ---- U = T V~ and W = T K~, one commit (bar_mma phase 1): A = T (K-major), B = V~ / K~ (MN-major)
    if (tid == 0) {
        tc_fence_after();
        const uint32_t idesc = idesc_f16_f32(128, 128, false, true);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const uint64_t da = sdesc_sw128(sbase + OFF_LT + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
            umma_f16(tmem + TM_U, da, sdesc_sw128(sbase + OFF_QV + kk * 2048, 16384, 1024), idesc, kk > 0);
            umma_f16(tmem + TM_W, da, sdesc_sw128(sbase + OFF_K + kk * 2048, 16384, 1024), idesc, kk > 0);
        }
        umma_commit(bar_mma);
        ++mma_commits;
    }
    mbar_wait(bar_mma, 1, ab, p.status, p.wait_limit_ns);
    if (tid == 0 && p.save) bulk_wait_read_all();  // the T store has read the tile W is staged in
    __syncthreads();
    if (ab->flag) goto teardown;
    tc_fence_after();
    if (tid == 0) GDN_TRACE_AT(6);
    // ---- W rows (warps 0-3) into the L area, U rows (warps 4-7) into the V~ area; bulk stores
    {
        uint8_t *dst = sm + (groupL ? OFF_LT : OFF_QV);
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
        tma_store_2d(&tmW, sm + OFF_LT, 0, y0);
        tma_store_2d(&tmW, sm + OFF_LT + 16384, 64, y0);
        bulk_commit();
    }
    if (tid == 128) {
        tma_store_2d(&tmU, sm + OFF_QV, 0, y0);
        tma_store_2d(&tmU, sm + OFF_QV + 16384, 64, y0);
        bulk_commit();
    }
    if (tid == 0) GDN_TRACE_AT(7);

teardown:
    // after an abort, loads and tensor-core work still in flight complete before shared memory and
    // TMEM go away (bounded waits that ignore the abort flag; immediate when nothing is pending)
    if (tid == 0) {
        mbar_wait_drain(bar_load, 0, p.wait_limit_ns);
        if (mma_commits > 0) mbar_wait_drain(bar_mma, (mma_commits - 1) & 1, p.wait_limit_ns);
    }
    if (tid == 128 && v_issued) mbar_wait_drain(bar_v, 0, p.wait_limit_ns);
    if (tid == 0 || tid == 128) bulk_wait_all();  // every bulk store issued by this CTA has completed
    if (tid == 0) GDN_TRACE_AT(8);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

}  // namespace

cudaError_t launch_chunk(const ChunkParams &p, const CUtensorMap &tmK, const CUtensorMap &tmV,
                         const CUtensorMap &tmQ, const CUtensorMap &tmW, const CUtensorMap &tmU,
                         const CUtensorMap &tmQt, const CUtensorMap &tmAqk, const CUtensorMap &tmAqkH,
                         const CUtensorMap &tmT, cudaStream_t s, bool pdl) {
    static SmemOnce once;
    cudaError_t e = raise_smem_once(once, gdn_chunk_kernel, static_cast<int>(SMEM_BYTES));
    if (e != cudaSuccess) return e;
    dim3 grid(p.NB, p.BH);
    return launch_k(gdn_chunk_kernel, grid, dim3(256), SMEM_BYTES, s, pdl, p, tmK, tmV, tmQ, tmW, tmU, tmQt, tmAqk,
                    tmAqkH, tmT);
}

}  // namespace gdn

GDN_TRACE_EXPORT(chunk)
