// gemm.cu — block-scaled W4A4 GEMM on the 5th-generation tensor cores:
// C[M x N] = alpha * sum_k deq(A[m,k]) * deq(W[n,k]), FP32 accumulation in
// tensor memory ("4.5 FP8 and NVFP4/MXFP4" §5: both operands FP4 on the
// Blackwell tensor cores; "FP4 quantization analysis: MXFP4 vs NVFP4" §3.3:
// FP4-specific operand re-layout feeding the GEMM).
//
// Operands come straight from fp4_quantize: packed E2M1 rows (K-major) and
// scales already in the 128x4 atom layout the MMA reads, so no re-layout
// pass exists.  alpha = s_gA * s_gW for NVFP4, 1 for MXFP4.  MXFP4 on
// 16-element blocks runs the NVFP4 (16-element block) instantiations with
// the MMA's scale type switched to E8M0 at run time (sf_e8m0) and alpha = 1.
//
// Prefill (M > 16): a persistent kernel over 128*CG x 256 output tiles, CG = 2
// (CTA pairs sharing one 2-SM MMA) once A spans more than 128 rows; see
// pgemm_kernel.  Its epilogue stores FP32, BF16, or C quantized again to
// MXFP4 / NVFP4 for the next layer (the QuTLASS-style fused epilogue of the
// same page, §3.3).  Decode (M <= 16): a weight-streaming split-K kernel with
// four MMA-issuing warps and a deterministic reduction; see decode_kernel.
// K is any multiple of 32: the last 256-wide K step of a tail reads zeros.
// Every wait is bounded (%globaltimer); a wait that gives up sets the device
// error word, the kernel stops issuing work, frees its TMEM and returns
// without storing.
#include <cudaTypedefs.h>

#include <atomic>
#include <mutex>
#include <set>
#include <type_traits>
#include <utility>

#include "encode.cuh"
#include "sm100.cuh"

namespace fp4 {

static __device__ unsigned int g_gemm_error;

// ---------------------------------------------------------------------------
// Persistent tiled kernel.  Each CTA (CG == 1) or CTA pair (CG == 2, one
// 2-SM MMA covering 256 rows of A) walks output tiles of 128*CG x 256 in
// M-fastest order, strided by the number of CTA groups, so the tiles resident
// at one time share the same W columns in L2.  Roles:
//   warp 0       TMA producer, runs ahead across tile boundaries: A rows of
//                this CTA, its share of the 256 W rows (all of them for
//                CG == 1, half for CG == 2) and the scale atoms (A: this CTA's
//                128 rows; W: all 256 rows, both CTAs), counted on the full
//                barrier of the group's leader CTA;
//   warp 1       TMEM allocation; in the leader CTA also the MMA issuer:
//                four K=64 block-scaled MMAs per stage once the stage's
//                scales are in TMEM, tcgen05.commit to free the stage (in
//                both CTAs);
//   warps 10-11  (leader CTA) scale copiers: tcgen05.cp of the stage's scale
//                atoms into TMEM, half each, then a commit that releases the
//                stage to the MMA issuer.  A tcgen05 instruction costs its
//                issuing thread tens of cycles, so copies issued from other
//                warps overlap the MMAs instead of queueing in front of them;
//   warps 2-9    epilogue: two warps per 32-lane quarter, each draining 128
//                accumulator columns into registers, then releasing the
//                accumulator (so the next tile's MMAs start) before scaling,
//                converting and storing.
template <int CG>
struct PCfg {
    static constexpr int BM = 128;                       // rows of A per CTA
    static constexpr int BN = 256;                       // output columns per tile
    static constexpr int BK = 256;                       // fp4 elements per stage
    static constexpr int B_ROWS = BN / CG;               // W rows loaded per CTA
    static constexpr int A_BYTES = BM * BK / 2;
    static constexpr int B_BYTES = B_ROWS * BK / 2;
    static constexpr int SFA_BYTES = 4 * 512;
    static constexpr int SFB_BYTES = 2 * 4 * 512;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
    static constexpr int STAGES = CG == 1 ? 4 : 5;
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + 256;
    static constexpr int NCOPY = 2;                      // scale-copier warps (10 and 11)
    static constexpr int THREADS = 384;
    static constexpr int TMEM_COLS = 512;
    static constexpr int SF_COL0 = 256;
    static constexpr int SF_STAGE_COLS = 48;
    static_assert(STAGE_BYTES % 1024 == 0, "stages must keep 1024-byte alignment for the 128-byte swizzle");
    static_assert(SF_COL0 + STAGES * SF_STAGE_COLS <= TMEM_COLS, "TMEM budget");
};

// Output modes of the prefill kernel.
enum { OUT_F32 = 0, OUT_BF16 = 1, OUT_MXFP4 = 2, OUT_NVFP4 = 3 };

struct PParams {
    const float *gA;
    const float *gW;
    void *C;             // fp32 / bf16 C, or the packed FP4 elements of C (M x N/2 bytes)
    int64_t ldc;
    // FP4 output (the product quantized again along N for the next layer):
    uint8_t *Cs;         // scales in the tile layout
    const float *gC;     // NVFP4: the given tensor scale of C
    int nkb4c;           // ceil(N / block / 4)
    int round_away, mx_floor;
    int M, N, K;
    int nkb4;
    int num_m_tiles, num_n_tiles;
    int sf_e8m0;         // FMT == NVFP4 only: E8M0 block scales (MXFP4 on 16-element blocks), alpha = 1
    uint64_t budget_ns;  // limit of every mbarrier wait
    int stall;           // failure-detection test: the producer issues no loads
};

template <int FMT, int OUT, int CG>
__global__ void __launch_bounds__(384, 1)
pgemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
             const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmSB, PParams p)
{
    using Cfg = PCfg<CG>;
    constexpr int KA = (FMT == FP4_MXFP4) ? 2 : 4;
    constexpr int STAGES = Cfg::STAGES;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGES * Cfg::STAGE_BYTES);
    // bars: full[S] empty[S] sfready[S] accfull accempty drain
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 3 * STAGES + 3);
    volatile uint32_t *abort_flag = tmem_slot + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = (CG == 2) ? cluster_ctarank() : 0u;
    const bool leader = rank == 0;
    const int group = blockIdx.x / CG, ngroups = gridDim.x / CG;
    const int num_tiles = p.num_m_tiles * p.num_n_tiles;
    const int nk = (p.K + Cfg::BK - 1) / Cfg::BK;  // a K tail reads zeros past K (TMA fill)

    const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + STAGES), sfr0 = smem_u32(bars + 2 * STAGES);
    const uint32_t accf = smem_u32(bars + 3 * STAGES), acce = smem_u32(bars + 3 * STAGES + 1);
    const uint32_t drainb = smem_u32(bars + 3 * STAGES + 2);
    // the leader's copies of the barriers every CTA of the group signals
    const uint32_t full0_lead = (CG == 2) ? mapa_shared(full0, 0) : full0;
    const uint32_t acce_lead = (CG == 2) ? mapa_shared(acce, 0) : acce;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; s++) {
            mbar_init(full0 + 8 * s, CG);   // one arrive.expect_tx per CTA of the group
            mbar_init(empty0 + 8 * s, 1);   // one tcgen05.commit
            mbar_init(sfr0 + 8 * s, Cfg::NCOPY);  // one commit per scale copier
        }
        mbar_init(accf, 1);
        mbar_init(drainb, 1 + Cfg::NCOPY);  // MMA issuer and copiers, once each at the end
        mbar_init(acce, 8 * CG);            // every epilogue warp of the group
        *abort_flag = 0u;
        fence_barrier_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmSA);
        tma_prefetch_desc(&tmSB);
    }
    if (warp == 1) {
        tmem_alloc_cg<CG>(smem_u32(tmem_slot), Cfg::TMEM_COLS);
        tmem_relinquish_cg<CG>();
    }
    tc_fence_before();
    if (CG == 2) cluster_sync(); else __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    grid_dep_launch();
    grid_dep_wait();  // operands may come from the preceding kernel

    if (warp == 0) {
        if (lane == 0 && !p.stall) {
            // ---------------- TMA producer ----------------
            const uint32_t tx = Cfg::A_BYTES + Cfg::B_BYTES + 3 * KA * 512;
            int it = 0;
            for (int t = group; t < num_tiles; t += ngroups) {
                const int mt = t % p.num_m_tiles, nt = t / p.num_m_tiles;
                const int arow = (mt * CG + (int)rank) * Cfg::BM;
                const int brow = nt * Cfg::BN + (int)rank * Cfg::B_ROWS;
                const int sfa_rb = mt * CG + (int)rank;  // 128-row blocks of the scale layouts
                const int sfb_rb0 = 2 * nt, sfb_rb1 = 2 * nt + 1;
                bool stop = false;
                for (int ks = 0; ks < nk; ks++, it++) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    if (!mbar_wait_bounded(empty0 + 8 * s, ph ^ 1, abort_flag, &g_gemm_error, p.budget_ns)) { stop = true; break; }
                    uint8_t *st = smem + s * Cfg::STAGE_BYTES;
                    const uint32_t fb = full0_lead + 8 * s;
                    if (CG == 1) mbar_arrive_expect_tx(fb, tx); else mbar_arrive_expect_tx_cluster(fb, tx);
                    tma_load_2d_cg<CG>(smem_u32(st), &tmA, ks * (Cfg::BK / 2), arow, fb);
                    tma_load_2d_cg<CG>(smem_u32(st + Cfg::A_BYTES), &tmB, ks * (Cfg::BK / 2), brow, fb);
                    const uint32_t ssf = smem_u32(st + Cfg::A_BYTES + Cfg::B_BYTES);
                    tma_load_3d_cg<CG>(ssf, &tmSA, 0, ks * KA, sfa_rb, fb);
                    tma_load_3d_cg<CG>(ssf + Cfg::SFA_BYTES, &tmSB, 0, ks * KA, sfb_rb0, fb);
                    tma_load_3d_cg<CG>(ssf + Cfg::SFA_BYTES + KA * 512, &tmSB, 0, ks * KA, sfb_rb1, fb);
                }
                if (stop) break;
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ---------------- MMA issuer (leader CTA) ----------------
            int it = 0, tile_i = 0;
            const uint16_t both = (uint16_t)((1u << CG) - 1u);
            // stage-0 descriptors; stages and K steps add to the 16-byte-unit
            // address field (offsets stay below 256 KB: no carry)
            const uint32_t sa0 = smem_u32(smem);
            const uint64_t adesc0 = smem_desc(sa0, 16, 1024, 2);
            const uint64_t bdesc0 = smem_desc(sa0 + Cfg::A_BYTES, 16, 1024, 2);
            for (int t = group; t < num_tiles; t += ngroups, tile_i++) {
                if (tile_i > 0 &&
                    !mbar_wait_bounded(acce, (uint32_t)((tile_i - 1) & 1), abort_flag, &g_gemm_error, p.budget_ns))
                    break;
                tc_fence_after();
                bool stop = false;
                for (int ks = 0; ks < nk; ks++, it++) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    // operands landed and the scale copiers' tcgen05.cp done
                    if (!mbar_wait_bounded(sfr0 + 8 * s, ph, abort_flag, &g_gemm_error, p.budget_ns)) { stop = true; break; }
                    tc_fence_after();
                    const uint64_t so = (uint64_t)((s * Cfg::STAGE_BYTES) >> 4);
                    const uint32_t tsfa = tmem + Cfg::SF_COL0 + s * Cfg::SF_STAGE_COLS;
                    const uint32_t tsfb = tsfa + 16;
#pragma unroll
                    for (int kk = 0; kk < 4; kk++) {
                        const uint64_t ad = adesc0 + so + 2 * kk;
                        const uint64_t bd = bdesc0 + so + 2 * kk;
                        const int atom = (FMT == FP4_MXFP4) ? (kk >> 1) : kk;
                        const uint32_t sfid = (FMT == FP4_MXFP4) ? (uint32_t)((kk & 1) * 2) : 0u;
                        const uint32_t idesc = idesc_blockscaled(Cfg::BM * CG, Cfg::BN, FMT == FP4_MXFP4 || p.sf_e8m0, sfid, sfid);
                        tc_mma_blockscaled_cg<FMT, CG>(tmem, ad, bd, idesc, (tsfa + 4 * atom) | (sfid << 30),
                                                       (tsfb + 8 * atom) | (sfid << 30), (ks | kk) ? 1u : 0u);
                    }
                    tc_commit_cg<CG>(empty0 + 8 * s, both);
                }
                if (stop && CG == 2) {
                    // the peer CTA's epilogue must not store after an abort
                    asm volatile("st.shared::cluster.u32 [%0], %1;\n\tfence.acq_rel.cluster;" ::"r"(
                                     mapa_shared(smem_u32((const void *)abort_flag), 1)),
                                 "r"(1u)
                                 : "memory");
                }
                // the accumulator is ready (or, after an abort, no MMA is left in flight)
                tc_commit_cg<CG>(accf, both);
                if (stop) break;
            }
            // TMEM is released only after every MMA and scale copy of the
            // group has completed, also on the abort path
            tc_commit_cg<CG>(drainb, 1);
            volatile uint32_t no_abort = 0;
            mbar_wait_bounded(drainb, 0, &no_abort, &g_gemm_error, p.budget_ns);
        }
        __syncwarp();
    } else if (warp >= 10) {
        // ---------------- scale copiers (leader CTA) ----------------
        if (lane == 0 && leader) {
            constexpr int APC = KA / Cfg::NCOPY;  // scale atoms per copier per stage
            const int c = warp - 10;
            const uint32_t sa0 = smem_u32(smem);
            const uint64_t sfadesc0 = smem_desc(sa0 + Cfg::A_BYTES + Cfg::B_BYTES, 0, 128, 0);
            const uint64_t sfbdesc0 = sfadesc0 + (Cfg::SFA_BYTES >> 4);
            int it = 0;
            bool stop = false;
            for (int t = group; t < num_tiles && !stop; t += ngroups) {
                for (int ks = 0; ks < nk; ks++, it++) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    // the stage's previous MMAs finished before it was reloaded
                    // (empty -> producer -> full), so its scale columns are free
                    if (!mbar_wait_bounded(full0 + 8 * s, ph, abort_flag, &g_gemm_error, p.budget_ns)) { stop = true; break; }
                    tc_fence_after();
                    const uint64_t so = (uint64_t)((s * Cfg::STAGE_BYTES) >> 4);
                    const uint32_t tsfa = tmem + Cfg::SF_COL0 + s * Cfg::SF_STAGE_COLS;
                    const uint32_t tsfb = tsfa + 16;
#pragma unroll
                    for (int q = 0; q < APC; q++) {
                        const int a = c * APC + q;
                        tc_cp_scale_atom_cg<CG>(tsfa + 4 * a, sfadesc0 + so + 32 * a);
                        tc_cp_scale_atom_cg<CG>(tsfb + 8 * a, sfbdesc0 + so + 32 * a);
                        tc_cp_scale_atom_cg<CG>(tsfb + 8 * a + 4, sfbdesc0 + so + 32 * (KA + a));
                    }
                    tc_commit_cg<CG>(sfr0 + 8 * s, 1);
                }
            }
            tc_commit_cg<CG>(drainb, 1);
        }
        __syncwarp();
    } else {
        // ---------------- epilogue: warps 2..9 ----------------
        constexpr bool BF16OUT = OUT == OUT_BF16;
        const int quarter = warp & 3;          // TMEM lanes this warp may read
        const int half = (warp - 2) >> 2;      // accumulator columns [128*half, 128*half + 128)
        const bool vec32 = BF16OUT ? (p.ldc % 16 == 0) : (p.ldc % 8 == 0);
        const bool aligned_c = (reinterpret_cast<uintptr_t>(p.C) & 31) == 0;
        int tile_i = 0;
        for (int t = group; t < num_tiles; t += ngroups, tile_i++) {
            bool ok = !*abort_flag && mbar_wait_bounded(accf, (uint32_t)(tile_i & 1), abort_flag, &g_gemm_error, p.budget_ns);
            ok = __all_sync(0xFFFFFFFFu, ok);
            if (!ok || *abort_flag) break;
            tc_fence_after();
            const int mt = t % p.num_m_tiles, nt = t / p.num_m_tiles;
            uint32_t r[128];
            const uint32_t base = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(half * 128);
            tmem_ld32(base + 0, r + 0);
            tmem_ld32(base + 32, r + 32);
            tmem_ld32(base + 64, r + 64);
            tmem_ld32(base + 96, r + 96);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (CG == 1) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(acce) : "memory");
                else mbar_arrive_cluster(acce_lead);
            }
            const float alpha = (FMT == FP4_NVFP4 && !p.sf_e8m0) ? __fmul_rn(*p.gA, *p.gW) : 1.0f;
            const int m = (mt * CG + (int)rank) * Cfg::BM + quarter * 32 + lane;
            const int n0 = nt * Cfg::BN + half * 128;
            if (OUT >= OUT_MXFP4) {
                // C quantized along N for the next layer: this thread's 128
                // columns are 4 units of 32 (encode.cuh, as in the quantize
                // kernels); rows past M (up to the tile layout's padding to
                // 128 rows) get zero scales and no elements.
                constexpr int QF = OUT == OUT_MXFP4 ? FP4_MXFP4 : FP4_NVFP4;
                const float sgc = (QF == FP4_NVFP4) ? *p.gC : 1.0f;
                const float six_sgc = __fmul_rn(6.0f, sgc);
                uint8_t *cq = static_cast<uint8_t *>(p.C);
                const bool in_layout = m < (p.M + 127) / 128 * 128;  // the scale tile layout's rows
#pragma unroll
                for (int u = 0; u < 4; u++) {
                    const int n = n0 + 32 * u;
                    if (n >= p.N || !in_layout) break;
                    float v[32];
#pragma unroll
                    for (int e = 0; e < 32; e++) v[e] = __uint_as_float(r[32 * u + e]);
                    scale_halves(v, alpha, alpha);
                    uint4 nib;
                    uint32_t sb = encode_unit<QF>(v, sgc, six_sgc, p.round_away, p.mx_floor, nib);
                    if (m < p.M)
                        *reinterpret_cast<uint4 *>(cq + (int64_t)m * (p.N / 2) + n / 2) = nib;
                    else
                        sb = 0;
                    if (QF == FP4_MXFP4)
                        p.Cs[scale_offset(m, n / 32, p.nkb4c)] = (uint8_t)sb;
                    else
                        *reinterpret_cast<uint16_t *>(p.Cs + scale_offset(m, n / 16, p.nkb4c)) = (uint16_t)sb;
                }
            } else if (m < p.M && n0 < p.N) {
                if (BF16OUT) {
                    __nv_bfloat16 *row = reinterpret_cast<__nv_bfloat16 *>(p.C) + (int64_t)m * p.ldc + n0;
                    const bool fast = vec32 && aligned_c && n0 + 128 <= p.N;
#pragma unroll
                    for (int c = 0; c < 8; c++) {
                        uint32_t w[8];
#pragma unroll
                        for (int e = 0; e < 8; e++) {
                            __nv_bfloat162 h = __floats2bfloat162_rn(__fmul_rn(__uint_as_float(r[16 * c + 2 * e]), alpha),
                                                                     __fmul_rn(__uint_as_float(r[16 * c + 2 * e + 1]), alpha));
                            w[e] = *reinterpret_cast<uint32_t *>(&h);
                        }
                        if (fast) {
                            st_global_v8(row + 16 * c, w);
                        } else {
#pragma unroll
                            for (int e = 0; e < 16; e++)
                                if (n0 + 16 * c + e < p.N)
                                    reinterpret_cast<uint16_t *>(row)[16 * c + e] = (uint16_t)(w[e >> 1] >> (16 * (e & 1)));
                        }
                    }
                } else {
                    float *row = reinterpret_cast<float *>(p.C) + (int64_t)m * p.ldc + n0;
                    const bool fast = vec32 && aligned_c && n0 + 128 <= p.N;
#pragma unroll
                    for (int c = 0; c < 16; c++) {
                        uint32_t w[8];
#pragma unroll
                        for (int e = 0; e < 8; e++) w[e] = __float_as_uint(__fmul_rn(__uint_as_float(r[8 * c + e]), alpha));
                        if (fast) {
                            st_global_v8(row + 8 * c, w);
                        } else {
#pragma unroll
                            for (int e = 0; e < 8; e++)
                                if (n0 + 8 * c + e < p.N) row[8 * c + e] = __uint_as_float(w[e]);
                        }
                    }
                }
            }
        }
    }

    tc_fence_before();
    if (CG == 2) cluster_sync(); else __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_cg<CG>(tmem, Cfg::TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------
// Decode kernel (M <= 16): the weight stream dominates, so the roles swap: a
// 128-row W tile is the MMA's M operand and the (up to 16) activation rows
// are N = 16.  Work is cut into (W tile, 256-wide K step) units, and each CTA
// accumulates the units it owns in TMEM (two buffers, alternating per tile;
// within a buffer one accumulator per issuing warp, added in warp order).
// Three ways to spread the tiles over the SMs (plan()):
//   * whole tiles (ntiles <= SMs, no spare SMs for a split): one CTA per
//     tile, C stored straight from the accumulator;
//   * cluster split: each tile's K range is cut into S = 2, 4 or 8 slices,
//     one CTA each, and the S CTAs form a thread-block cluster.  Every CTA
//     leaves its 128 x 16 fp32 partial in shared memory and the cluster's
//     first CTA sums them in rank order over distributed shared memory;
//   * global split (very few tiles, or more tiles than SMs: stream-K over
//     the units): partials go to a workspace and are summed in CTA order,
//     either by the last CTA of the tile (per-tile arrival counters) or by
//     reduce_kernel.
namespace decode {

constexpr int BMW = 128, BNA = 16, BK = 256;
constexpr int W_BYTES = BMW * BK / 2;        // 16 KB
constexpr int SFW_BYTES = 4 * 512;
constexpr int SFA_BYTES = 4 * 512;
constexpr int TMEM_COLS = 512;
constexpr int NI = 4;                        // MMA issuer warps (warps 1, 6, 7, 8) at most
constexpr int SF_STAGE_COLS = 32;            // W scales 16 cols, activation scales 16 cols
constexpr int MAX_CLUSTER = 8;               // portable cluster size
// A cluster split's CTAs each read all of x for the NVFP4 tensor maximum
// while x (M x K bf16) is at most this large, instead of exchanging their
// K slices' maxima (a cross-CTA wait that costs more than the extra reads).
constexpr int64_t X_LOCAL_AMAX_BYTES = int64_t(64) << 10;

// Stage and tensor-memory layout of a decode_kernel variant.  A stage holds
// [W tile 128 x 256 | activation rows NB x 256 | W scale atoms | activation
// scale atoms], the rows 128 bytes each in the 128-byte swizzle.  NB = 16
// (1 + ND): the residual variant's ND groups of 16 more rows carry the
// sparse residual lane's values, split into terms the block-scaled MMA
// multiplies exactly, through the same MMA as the activations.  Tensor
// memory: NBUF accumulator buffers of NIS issuers x NB columns, then STAGES x
// 32 columns of scales.  Issuer j takes the units i = j (mod NIS); STAGES is
// a multiple of NIS so that a stage is always consumed by the same issuer:
// an issuer then waits for every phase of its stages' barriers in turn, which
// is what their parity waits need (a barrier two phases further than its
// waiter last saw reads as ready).
template <int ND, int NSTAGES, int NISSUERS, int NQX>
struct DCfg {
    static constexpr int STAGES = NSTAGES;
    static constexpr int NIS = NISSUERS;
    static constexpr int NQ = 4 + NQX;  // fused variants: activation quantizer warps (2-5 and NQX more)
    static constexpr int NB = BNA * (1 + ND);
    static constexpr int A_BYTES = NB * BK / 2;
    static constexpr int STAGE_BYTES = W_BYTES + A_BYTES + SFW_BYTES + SFA_BYTES;
    static constexpr int NBUF = ND ? 1 : 2;  // the residual variant runs one tile segment per CTA
    static constexpr int SF_COL0 = NBUF * NIS * NB;
    static_assert(STAGES % NIS == 0 && NIS <= NI, "a stage is always consumed by the same issuer");
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + 512;
    static_assert(STAGE_BYTES % 1024 == 0, "stages keep the 1024-byte alignment of the 128-byte swizzle");
    static_assert(SF_COL0 + STAGES * SF_STAGE_COLS <= TMEM_COLS, "TMEM budget");
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
    static_assert(NB <= 128, "one 128-row scale atom covers the activation rows");
};
// fp4_gemm's and fp4_linear's decode kernels: 8 stages of 22 KB, 4 issuers,
// 8 quantizer warps (fused: 13 warps in all, one per stage: with 7 quantizers
// and so 12 warps, the warp writing two stages held M = 16 back by 2.4 to
// 3.5 us, more than the spills of 13 warps cost)
using DPlain = DCfg<0, 8, 4, 4>;
// the residual lane (fp4_linear_residual): 4 groups of term rows, 6 stages
// of 30 KB, 3 issuers, 8 quantizer warps (12 warps in all).
// E8M0-scaled terms have two significant bits, so a bf16 value takes up to 4
// (MXFP4, MXFP4_16); E4M3-scaled terms have four, so 2, in one of two bands
// of a row's scale (NVFP4)
template <int QFMT>
using DRes = DCfg<4, 6, 3, 4>;
struct Params {
    float *ws;           // partials: [G][maxseg][128][16]
    // Fused reduction (counters != nullptr): per-tile arrival counters, zero
    // on entry; the last CTA to finish a tile sums its partials and stores C.
    unsigned *counters;
    const float *gA, *gW;
    void *C;
    int64_t ldc;
    int bf16out;
    int sf_e8m0;         // FMT == NVFP4 only: E8M0 block scales (MXFP4 on 16-element blocks), alpha = 1
    uint64_t budget_ns;  // limit of every mbarrier wait
    int stall;           // failure-detection test: the producer issues no loads
    int N, M, K;
    int nk;              // ceil(K / BK); the last K step of a tail reads zeros past K
    int ntiles;          // ceil(N / 128)
    int G;               // CTAs
    int maxseg;
    int csize;           // > 1: the CTAs of a tile form a cluster of csize and reduce through DSMEM
    // Stream W before waiting for the preceding kernel.  Only when that
    // kernel triggers its dependents after its own wait (the decode
    // activation quantizer, or the fused kernel of an earlier fp4_linear), so
    // every earlier kernel, whatever wrote W, has finished.
    int w_before_wait;
    // Fused activation quantization (fp4_linear): bf16 x, M x K, row stride
    // ldx elements; gA null = the NVFP4 tensor scale is computed from x.
    const uint16_t *x;
    int64_t ldx;
    int xwide;           // x and its row stride are 32-byte aligned: 32-byte loads
    float ck;            // RN(1/sqrt(k)) of the rotation
    int round_away, mx_floor;
};

__host__ __device__ inline int64_t unit_begin(int c, int64_t U, int G) { return (int64_t)c * U / G; }
// The CTA whose unit range contains unit u.
__host__ __device__ inline int unit_owner(int64_t u, int64_t U, int G) { return (int)(((u + 1) * G + U - 1) / U) - 1; }

// C[m][n] for the m < M activation rows of one output row n.
FP4_DEV void store_row(const Params &p, int n, const float *acc, float alpha)
{
#pragma unroll
    for (int m = 0; m < BNA; m++) {
        if (m >= p.M) break;
        const float v = __fmul_rn(acc[m], alpha);
        if (p.bf16out)
            reinterpret_cast<__nv_bfloat16 *>(p.C)[(int64_t)m * p.ldc + n] = __float2bfloat16_rn(v);
        else
            reinterpret_cast<float *>(p.C)[(int64_t)m * p.ldc + n] = v;
    }
}

// Threads: warp 0 loads, warps 1 and 6 .. 4 + NIS issue MMAs (NIS issuers:
// 1, 6, 7, 8 for four), warps 2-5 drain the accumulators (warp w may read
// TMEM lanes 32 (w % 4) .. + 31).  The fused variants (fp4_linear,
// fp4_linear_residual) add NQX warps after the issuers: with warps 2-5 they
// quantize the activations into the stages before the accumulators are
// drained.  Thirteen warps cap a thread at 128 registers (four of them
// share one SM sub-partition's 16K) and the NVFP4 quantizers spill; twelve
// (the residual variant, one issuer fewer) allow 168.
__host__ __device__ constexpr int decode_threads(bool fused, int nis, int nqx)
{
    return 32 * (6 + nis - 1 + (fused ? nqx : 0));
}

// Quantizer warp index of warp w (fused variants): warps 2-5 -> 0-3, the
// warps after the issuers -> 4, 5, ...
FP4_DEV int quantizer_index(int warp, int nis) { return warp <= 5 ? warp - 2 : warp - nis - 1; }

// Named barrier over the NQ quantizer warps (id 2; id 1 is the epilogue's).
template <int NQ>
FP4_DEV void quantizers_sync() { asm volatile("bar.sync 2, %0;" ::"n"(NQ * 32) : "memory"); }

// True for all four epilogue warps (2-5) iff v holds in every one of their
// threads: one abort decision for warps that then take the same sequence of
// named barriers (a warp that left the loop alone would strand the others
// at the reduction's bar.sync).
FP4_DEV bool epilogue_all(bool v)
{
    int r;
    asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.s32 q, %1, 0;\n\tbar.red.and.pred p, 1, 128, q;\n\t"
                 "selp.s32 %0, 1, 0, p;\n\t}"
                 : "=r"(r)
                 : "r"(v ? 1 : 0)
                 : "memory");
    return r != 0;
}

// Makes this thread's generic-proxy shared-memory writes visible to the
// tensor cores' (async-proxy) reads that follow a barrier.
FP4_DEV void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

FP4_DEV void mbar_arrive_local(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Arrive on a barrier of another CTA of the cluster, ordering this thread's
// earlier shared::cluster stores before it (release at cluster scope).
FP4_DEV void mbar_arrive_remote_release(uint32_t bar_cluster)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}

// Bounded wait with acquire at cluster scope (sees the stores that remote
// arrivals released).
FP4_DEV bool mbar_wait_cluster_bounded(uint32_t bar, uint32_t parity, volatile uint32_t *abort, unsigned int *err_word,
                                       uint64_t budget_ns)
{
    const uint64_t t0 = globaltimer();
    for (;;) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(bar), "r"(parity)
            : "memory");
        if (ok) return true;
        if (*abort) return false;
        if (globaltimer() - t0 > budget_ns) {
            *abort = 1u;
            atomicOr(err_word, 1u);
            return false;
        }
    }
}

FP4_DEV void st_shared_cluster_f32(uint32_t addr_cluster, float v)
{
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr_cluster), "f"(v) : "memory");
}

// Raw bf16 bytes of unit column j of activation row m (zeros for a row at or
// past M, or a column at or past K: they quantize to zero codes and zero
// scales, finite as the product's K tail needs).  Read through L2 only: x
// may be the output of the kernel this one overlapped.
FP4_DEV void ld_cg_v8(const void *ptr, uint4 &a, uint4 &b)
{
    asm volatile("ld.global.cg.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(a.x), "=r"(a.y), "=r"(a.z), "=r"(a.w), "=r"(b.x), "=r"(b.y), "=r"(b.z), "=r"(b.w)
                 : "l"(ptr));
}

FP4_DEV void fetch_act_unit(const Params &p, int m, int j, uint4 *raw)
{
    if (m < p.M && j < p.K / 32) {
        const uint4 *src = reinterpret_cast<const uint4 *>(p.x + (int64_t)m * p.ldx + (int64_t)j * 32);
        if (p.xwide) {  // two 32-byte loads: a full sector per lane
            ld_cg_v8(src, raw[0], raw[1]);
            ld_cg_v8(src + 2, raw[2], raw[3]);
            return;
        }
#pragma unroll
        for (int c = 0; c < 4; c++) raw[c] = __ldcg(src + c);
    } else {
#pragma unroll
        for (int c = 0; c < 4; c++) raw[c] = make_uint4(0, 0, 0, 0);
    }
}

// ---- the sparse residual lane in the product ----------------------------------
// "Portable FP4 quantization (TransFP4)" §2.3 Eq.(3): with both operands
// rotated by the same H, C = Q(A - R) Q_W^T + R Q_W^T, R holding one value per
// 32-element unit of a row (its largest rotated value, as bf16).  The second
// term rides on the tensor cores: each residual r is split into ND terms
// that the block-scaled MMA represents exactly (one nonzero element in its
// block, whose scale carries the magnitude), placed at the residual's K
// position in ND extra groups of 16 activation rows, so one MMA with
// N = 16 (1 + ND) multiplies the weight tile with the activations and with
// every term.  The epilogue adds the term rows to the residual sum.

// E8M0-scaled terms (MXFP4, MXFP4_16): r as at most 4 terms sign * {1, 1.5}
// * 2^e, each the next two significant bits of what is left (E2M1 codes 2 and
// 3 under the E8M0 scale byte e + 127); bf16 has 8 significant bits, so 4
// terms leave nothing.  Terms below 2^-126 (fp32 subnormal) are dropped.
FP4_DEV void residual_terms_e8m0(float r, uint32_t *code, uint32_t *sbyte)
{
    float rem = r;
#pragma unroll
    for (int d = 0; d < 4; d++) {
        const uint32_t u = __float_as_uint(rem);
        const uint32_t ef = (u >> 23) & 0xFFu;
        if (ef == 0) {
            code[d] = 0;
            sbyte[d] = 0;
            continue;
        }
        const float t = __uint_as_float(u & 0xFFC00000u);  // sign, exponent, first mantissa bit
        rem = __fsub_rn(rem, t);                             // exact: t is a prefix of rem
        code[d] = (((u >> 22) & 1u) ? 3u : 2u) | ((u >> 28) & 8u);
        sbyte[d] = ef;  // 2^(ef - 127): the term's exponent as an E8M0 byte
    }
}

// E4M3-scaled terms (NVFP4): u = r / 2^E as at most 2 E4M3 values, the
// nearest one, then the nearest to what is left (which has at most 4
// significant bits: the rounding error of an 8-bit value at 4 bits), each an
// element +-1 (E2M1 code 2) under that block scale.  Exact while the terms
// stay within E4M3's range (see the row exponent below).
FP4_DEV void residual_terms_e4m3(float u, uint32_t *code, uint32_t *sbyte)
{
#pragma unroll
    for (int d = 0; d < 2; d++) {
        const uint32_t b = e4m3_rn(fabsf(u));
        const float v = e4m3_to_f32(b);
        sbyte[d] = b;
        code[d] = b ? (2u | ((__float_as_uint(u) >> 28) & 8u)) : 0u;
        u = __fsub_rn(u, copysignf(v, u));  // exact: both are multiples of u's last bit
    }
}

// Row exponent E0 of the NVFP4 terms: with e the exponent of the row's
// largest residual magnitude, E0 = e - 7 puts every u = r / 2^E0 below 256
// (inside E4M3's 448).  Two E4M3 terms of u are exact while the second one's
// last bit, 2^(e(r) - 7 - E0), stays at or above E4M3's smallest step 2^-9,
// i.e. for |r| >= 2^(E0 - 2): band 0.  Smaller residuals go to band 1, the
// same terms of r / 2^(E0 - 10), exact down to 2^(E0 - 12) = 2^(e - 19); below
// that (19 binades under the row's largest) the terms are E4M3 roundings.
// E0 is clamped so that both bands' factors stay normal floats.
constexpr int RES_BAND_SHIFT = 10;
FP4_DEV int residual_row_exponent(float rowmax)
{
    if (!(rowmax > 0.0f)) return 0;
    int e = (int)((__float_as_uint(rowmax) >> 23) & 0xFF) - 127;
    e -= 7;
    return e < -126 + RES_BAND_SHIFT ? -126 + RES_BAND_SHIFT : (e > 126 ? 126 : e);
}

// max |H_k x| over the unit columns [j0, j1) of every activation row,
// reduced over the NQ quantizer warps (all of them call it; every one gets
// the result).  j0 and j1 are multiples of k / 32, and consecutive lanes hold
// consecutive units of a row, so a rotation chunk lies in neighbouring lanes.
// RES: the maximum is that of the FP4 stream (each unit's residual value
// removed), and rowmax[m] (shared, zero on entry, float bits) receives the
// largest residual magnitude of row m.
template <int HK, bool RES, int NQ>
FP4_DEV float act_amax(const Params &p, int j0, int j1, int qw, int lane, float *red, unsigned *rowmax)
{
    const int ncols = j1 - j0;
    const int total = p.M * ncols;
    constexpr int U = 4;  // units per lane and trip, loads issued together
    float mx = 0.0f;
    for (int base = qw * 32 * U; base < total; base += NQ * 32 * U) {
        uint4 raw[U][4];
        int mrow[U];
#pragma unroll
        for (int i = 0; i < U; i++) {
            const int u = base + i * 32 + lane;
            mrow[i] = u < total ? u / ncols : p.M;
            fetch_act_unit(p, mrow[i], j0 + (u < total ? u - mrow[i] * ncols : 0), raw[i]);
        }
#pragma unroll
        for (int i = 0; i < U; i++) {
            float v[32];
            unpack_unit(raw[i], v);
            if (HK) fwht_unit<HK>(v, p.ck, lane);
            if (RES) {
                const uint32_t w = extract_residual(v);
                if (mrow[i] < p.M) atomicMax(rowmax + mrow[i], __float_as_uint(fabsf(bf16lo(w))));
            }
            mx = fmaxf(mx, absmax_tree<32>(v));
        }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
    if (lane == 0) red[qw] = mx;
    quantizers_sync<NQ>();
    float t = red[0];
#pragma unroll
    for (int w = 1; w < NQ; w++) t = fmaxf(t, red[w]);
    return t;
}

// The fused activation quantizer, one warp: for every unit i of this CTA
// whose stage s = i % STAGES has s % NQ == qw (its K step; a CTA's units may
// run over into the next tile), once the stage's previous MMAs are done,
// encodes the M x 256 activation slice of that K step into stage s exactly
// as the TMA would have
// placed fp4_quantize's output there (nibble rows of 128 bytes in the
// 128-byte swizzle; scales in the tile layout's atoms), then arrives on the
// stage's activation barrier.  Every use of a stage is written by the same
// warp, in order, so its wait for the stage's previous use always targets
// the phase after the last one it saw: a parity wait two phases behind would
// read as complete (a warp taking units i = qw (mod NQ) with NQ != STAGES
// waited for use 2 of a stage before use 0 was consumed).  Rows past M keep the zeros written at kernel
// start.  RES: each unit's residual value leaves the FP4 stream (as
// fp4_quantize_residual takes it) and its terms go to rows 16 d + m,
// d = 1 .. ND, at the residual's position (rexp[m]: the NVFP4 row exponent).
// Returns false after an abort.
template <int QFMT, int HK, bool RES, typename Cfg>
FP4_DEV bool quantize_act_stages(const Params &p, uint8_t *smem, uint32_t aready0, uint32_t empty0, int n_units,
                                 int t_first, int ks_first, int qw, int lane, float sg, const int *rexp,
                                 const NvScaleTables *tab, volatile uint32_t *abort_flag)
{
    constexpr int ND = Cfg::NB / BNA - 1;
    constexpr int R = BNA * 8 / 32;  // units per lane of one K step (16 rows x 8 units)
    const float six_sg = __fmul_rn(6.0f, sg);
    const int nwork = p.M * 8;  // units of one K step: (row m, column cu = 0..7)
    for (int i = 0; i < n_units; i++) {
        const int s = i % Cfg::STAGES;
        if (s % Cfg::NQ != qw) continue;
        const uint32_t ph = (uint32_t)((i / Cfg::STAGES) & 1);
        const int j0 = (int)(((int64_t)t_first * p.nk + ks_first + i) % p.nk) * 8;  // K step of unit i
        // Load and encode first, into registers; only the stores wait for the
        // stage to be free, so the loads' latency overlaps the MMAs of the
        // stage's previous use.
        uint4 raw[R][4];
#pragma unroll
        for (int r = 0; r < R; r++) {
            const int w = r * 32 + lane;
            if (r * 32 < nwork) fetch_act_unit(p, w < nwork ? w >> 3 : p.M, j0 + (w & 7), raw[r]);
        }
        uint4 nib[R];
        uint32_t sb[R];
        // residual lane, per unit: the terms' E2M1 codes (4 bits each) and the
        // residual's index << 16, and the terms' scale bytes (8 bits each)
        uint32_t tcodes[R], tscales[R];
#pragma unroll
        for (int r = 0; r < R; r++) {
            if (r * 32 >= nwork) break;  // warp-uniform
            const int w = r * 32 + lane;
            const int m = w >> 3;
            float v[32];
            unpack_unit(raw[r], v);
            if (HK) fwht_unit<HK>(v, p.ck, lane);
            uint32_t rw = 0;
            if (RES) rw = extract_residual(v);
            sb[r] = encode_unit<QFMT>(v, sg, six_sg, p.round_away, p.mx_floor, nib[r], tab);
            if (RES) {
                const float rv = bf16lo(rw);
                uint32_t code[ND > 0 ? ND : 1], sbyte[ND > 0 ? ND : 1];
                if (QFMT == FP4_NVFP4) {
                    // band 0 (rows 16-47) or band 1 (rows 48-79) of the row's scale
                    const int E0 = w < nwork ? rexp[m] : 0;
                    const bool hi = fabsf(rv) >= exp2i(E0 - 2);
                    uint32_t tc[2], ts[2];
                    residual_terms_e4m3(__fmul_rn(rv, exp2i(hi ? -E0 : RES_BAND_SHIFT - E0)), tc, ts);
#pragma unroll
                    for (int d = 0; d < 2; d++) {
                        code[d] = hi ? tc[d] : 0u;
                        sbyte[d] = hi ? ts[d] : 0u;
                        code[2 + d] = hi ? 0u : tc[d];
                        sbyte[2 + d] = hi ? 0u : ts[d];
                    }
                } else {
                    residual_terms_e8m0(rv, code, sbyte);
                }
                tcodes[r] = rw & 0x1F0000u;
                tscales[r] = 0;
#pragma unroll
                for (int d = 0; d < ND; d++) {
                    tcodes[r] |= code[d] << (4 * d);
                    tscales[r] |= sbyte[d] << (8 * d);
                }
            }
        }
        if (!mbar_wait_bounded(empty0 + 8 * s, ph ^ 1, abort_flag, &g_gemm_error, p.budget_ns)) return false;
        uint8_t *st = smem + s * Cfg::STAGE_BYTES;
        uint8_t *sa = st + W_BYTES;
        uint8_t *sfa = st + W_BYTES + Cfg::A_BYTES + SFW_BYTES;
#pragma unroll
        for (int r = 0; r < R; r++) {
            if (r * 32 >= nwork) break;  // warp-uniform
            const int w = r * 32 + lane;
            if (w >= nwork) continue;
            const int m = w >> 3, cu = w & 7;
            *reinterpret_cast<uint4 *>(sa + m * 128 + ((cu ^ (m & 7)) << 4)) = nib[r];
            if (QFMT == FP4_MXFP4)
                sfa[(cu >> 2) * 512 + m * 16 + (cu & 3)] = (uint8_t)sb[r];
            else
                *reinterpret_cast<uint16_t *>(sfa + (cu >> 1) * 512 + m * 16 + 2 * (cu & 1)) = (uint16_t)sb[r];
            if (RES) {
                const int idx = (int)(tcodes[r] >> 16);
#pragma unroll
                for (int d = 0; d < ND; d++) {
                    const int Rw = BNA * (d + 1) + m;  // Rw & 7 == m & 7
                    const uint32_t code = (tcodes[r] >> (4 * d)) & 0xFu, sbyte = (tscales[r] >> (8 * d)) & 0xFFu;
                    uint32_t wds[4] = {0u, 0u, 0u, 0u};
#pragma unroll
                    for (int q = 0; q < 4; q++)
                        if (q == (idx >> 3)) wds[q] = code << (4 * (idx & 7));
                    *reinterpret_cast<uint4 *>(sa + Rw * 128 + ((cu ^ (m & 7)) << 4)) =
                        make_uint4(wds[0], wds[1], wds[2], wds[3]);
                    const int rb = (Rw & 31) * 16 + (Rw >> 5) * 4;  // row's bytes in a scale atom
                    if (QFMT == FP4_MXFP4)
                        sfa[(cu >> 2) * 512 + rb + (cu & 3)] = (uint8_t)sbyte;
                    else  // two 16-element blocks: the term's block takes the scale, the other 0
                        *reinterpret_cast<uint16_t *>(sfa + (cu >> 1) * 512 + rb + 2 * (cu & 1)) =
                            (uint16_t)(sbyte << (8 * (idx >> 4)));
                }
            }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive_local(aready0 + 8 * s);
    }
    return true;
}

// C[m][n] for the m < M activation rows of one output row n, from the
// activation sum and the residual lane's sum: RN(alpha acc) + RN(aR[m] racc).
FP4_DEV void store_row_res(const Params &p, int n, const float *acc, const float *racc, float alpha, const float *aR)
{
#pragma unroll
    for (int m = 0; m < BNA; m++) {
        if (m >= p.M) break;
        const float v = __fadd_rn(__fmul_rn(acc[m], alpha), __fmul_rn(racc[m], aR[m]));
        if (p.bf16out)
            reinterpret_cast<__nv_bfloat16 *>(p.C)[(int64_t)m * p.ldc + n] = __float2bfloat16_rn(v);
        else
            reinterpret_cast<float *>(p.C)[(int64_t)m * p.ldc + n] = v;
    }
}

// QFMT: the operands' format (MXFP4_16 runs the 16-element block-scaled MMA,
// FMT below, with E8M0 scales).  FUSED: fp4_linear's single-launch form,
// which quantizes the activations itself (HK: their rotation) and needs a
// work split without tiles cut between CTAs outside a cluster; otherwise A
// comes quantized (fp4_gemm).  RES (fused only): the sparse residual lane in
// the product (fp4_linear_residual), one tile segment per CTA.
template <int QFMT, int HK, bool FUSED, bool RES>
__global__ void __launch_bounds__(decode_threads(FUSED, std::conditional<RES, DRes<QFMT>, DPlain>::type::NIS,
                                                 std::conditional<RES, DRes<QFMT>, DPlain>::type::NQ - 4),
                                  1)
decode_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmA,
              const __grid_constant__ CUtensorMap tmSW, const __grid_constant__ CUtensorMap tmSA, Params p)
{
    static_assert(FUSED || !RES, "the residual lane needs the fused activation quantizer");
    using Cfg = typename std::conditional<RES, DRes<QFMT>, DPlain>::type;
    constexpr int STAGES = Cfg::STAGES, STAGE_BYTES = Cfg::STAGE_BYTES, A_BYTES = Cfg::A_BYTES, NB = Cfg::NB;
    constexpr int NIS = Cfg::NIS;
    constexpr int ND = NB / BNA - 1;
    constexpr int FMT = QFMT == FP4_MXFP4 ? FP4_MXFP4 : FP4_NVFP4;
    constexpr int KA = (FMT == FP4_MXFP4) ? 2 : 4;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE_BYTES);
    // bars: full[S] (TMA bytes), empty[S], aready[S] (fused: the stage's
    // activations written), accfull[2], accempty[2], drain, amax (fused)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 3 * STAGES + 6);
    __shared__ volatile unsigned s_last;
    __shared__ float s_red[Cfg::NQ];        // fused: per-warp maxima
    __shared__ NvScaleTables s_tab;         // fused NVFP4: block-scale factors for s_g
    __shared__ float s_amax[MAX_CLUSTER];   // fused: the cluster CTAs' maxima, by rank
    __shared__ float s_sg;                  // fused: the activations' tensor scale
    __shared__ unsigned s_rowmax[BNA];      // residual lane, NVFP4: largest residual of each row (float bits)
    __shared__ int s_rexp[BNA];             // ... and its row exponent
    volatile uint32_t *abort_flag = tmem_slot + 1;
    // cluster split: this CTA's 128 x 16 partial, [4][128][4] floats (16-byte
    // groups of one row's columns 4q..4q+3), in stage 0's W buffer, which no
    // load or MMA touches once the accumulator is complete; the residual
    // variant's residual partial follows it in the same buffer
    float4 *part = reinterpret_cast<float4 *>(smem);

    // The fused kernels let the next launch start only after their own wait
    // (below): by then every kernel before this one has finished, so the next
    // one may stream static weights at once.
    if (!FUSED) grid_dep_launch();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x;
    const int64_t U = (int64_t)p.ntiles * p.nk;
    // This CTA's units [u0, u1): 32-bit divisions when the products fit (every
    // decode shape), 64-bit ones otherwise; the weight stream waits on them.
    int64_t u0, u1;
    int t_first, nseg_last;
    if ((uint64_t)U * (uint64_t)p.G < (1ull << 32)) {
        const uint32_t Uu = (uint32_t)U, Gu = (uint32_t)p.G, nk = (uint32_t)p.nk;
        const uint32_t a = (uint32_t)c * Uu / Gu, b = (uint32_t)(c + 1) * Uu / Gu;
        u0 = a;
        u1 = b;
        t_first = (int)(a / nk);
        nseg_last = (int)((b - 1) / nk);
    } else {
        u0 = unit_begin(c, U, p.G);
        u1 = unit_begin(c + 1, U, p.G);
        t_first = (int)(u0 / p.nk);
        nseg_last = (int)((u1 - 1) / p.nk);
    }
    // The loops below run on single threads, where integer latency is not
    // hidden: positions advance incrementally instead of by division.
    const int n_units = (int)(u1 - u0);
    const int ks_first = (int)(u0 - (int64_t)t_first * p.nk);
    const int nseg = nseg_last - t_first + 1;
    const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + STAGES), aready0 = smem_u32(bars + 2 * STAGES);
    const uint32_t accf0 = smem_u32(bars + 3 * STAGES), acce0 = smem_u32(bars + 3 * STAGES + 2);
    const uint32_t drainb = smem_u32(bars + 3 * STAGES + 4);
    const uint32_t amaxb = smem_u32(bars + 3 * STAGES + 5);
    const uint32_t tx = FUSED ? W_BYTES + KA * 512 : W_BYTES + A_BYTES + 2 * KA * 512;
    const int npre = n_units < STAGES ? n_units : STAGES;
    const uint32_t smem0 = smem_u32(smem);
    // NIS issuers: a tcgen05 instruction costs its issuing thread tens of
    // cycles, far longer than the tensor pipe needs for a skinny MMA, so NIS
    // warps take the units i = j (mod NIS) and accumulate them in their own
    // accumulators, which the epilogue adds in issuer order.  Every issuer
    // commits once per tile segment (also one that owns no unit of it), so
    // the segment barrier counts NIS arrivals.

    auto advance = [&](int &t, int &ks) {
        if (++ks == p.nk) {
            ks = 0;
            ++t;
        }
    };
    auto load_w = [&](int t, int ks, int st_i) {
        const uint32_t st = smem0 + st_i * STAGE_BYTES;
        const uint32_t fb = full0 + 8 * st_i;
        tma_load_2d(st, &tmW, ks * (BK / 2), t * BMW, fb);
        tma_load_3d(st + W_BYTES + A_BYTES, &tmSW, 0, ks * KA, t, fb);
    };
    auto load_a = [&](int ks, int st_i) {
        const uint32_t st = smem0 + st_i * STAGE_BYTES;
        const uint32_t fb = full0 + 8 * st_i;
        tma_load_2d(st + W_BYTES, &tmA, ks * (BK / 2), 0, fb);
        tma_load_3d(st + W_BYTES + A_BYTES + SFW_BYTES, &tmSA, 0, ks * KA, 0, fb);
    };

    if (threadIdx.x == 0) {
        tma_prefetch_desc(&tmW);
        tma_prefetch_desc(&tmSW);
        // the stages' TMA barriers first: with static weights the weight
        // stream starts before anything else is set up
        for (int s = 0; s < STAGES; s++) mbar_init(full0 + 8 * s, 1);
        fence_barrier_init();
        if (!p.stall && p.w_before_wait) {
            int t = t_first, ks = ks_first;
            for (int i = 0; i < npre; i++) {
                mbar_arrive_expect_tx(full0 + 8 * i, tx);
                load_w(t, ks, i);
                advance(t, ks);
            }
        }
        for (int s = 0; s < STAGES; s++) {
            mbar_init(empty0 + 8 * s, 1);
            mbar_init(aready0 + 8 * s, 1);  // fused: the stage's quantizer warp
        }
        for (int b = 0; b < 2; b++) {
            mbar_init(accf0 + 8 * b, NIS);
            mbar_init(acce0 + 8 * b, 4);  // one arrival per epilogue warp
        }
        mbar_init(drainb, NIS);
        mbar_init(amaxb, p.csize);  // fused, computed s_g: one arrival per CTA of the cluster
        *abort_flag = 0u;
        fence_barrier_init();
        if (!FUSED) {
            tma_prefetch_desc(&tmA);
            tma_prefetch_desc(&tmSA);
        }
        // Without the static-weights promise the weight stream starts after
        // the wait for the preceding kernel (which may have written W), while
        // warp 1 allocates tensor memory.
        if (!p.stall && !p.w_before_wait) {
            grid_dep_wait();
            int t = t_first, ks = ks_first;
            for (int i = 0; i < npre; i++) {
                mbar_arrive_expect_tx(full0 + 8 * i, tx);
                load_w(t, ks, i);
                advance(t, ks);
            }
        }
    }
    if (threadIdx.x < BNA) s_rowmax[threadIdx.x] = 0u;
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
        tmem_relinquish();
    }
    if (FUSED) {
        // activation rows past M are never written by the quantizers: zero
        // every stage's activation rows and scale atoms once
        for (int s = 0; s < STAGES; s++) {
            uint4 *a4 = reinterpret_cast<uint4 *>(smem + s * STAGE_BYTES + W_BYTES);
            uint4 *sf4 = reinterpret_cast<uint4 *>(smem + s * STAGE_BYTES + W_BYTES + A_BYTES + SFW_BYTES);
            for (int i = threadIdx.x; i < A_BYTES / 16; i += blockDim.x) a4[i] = make_uint4(0, 0, 0, 0);
            for (int i = threadIdx.x; i < SFA_BYTES / 16; i += blockDim.x) sf4[i] = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
    }
    tc_fence_before();
    // fused cluster split with the tensor maximum exchanged: the amax
    // barriers of every CTA are initialised before any CTA arrives on a peer's
    const bool amax_exchange = FUSED && QFMT == FP4_NVFP4 && p.csize > 1 &&
                               (RES || (!p.gA && (int64_t)p.M * p.K * 2 > X_LOCAL_AMAX_BYTES));
    if (amax_exchange) cluster_sync(); else __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0 && !p.stall) {
            grid_dep_wait();
            int t = t_first, ks = ks_first;
            if (!FUSED) {
                for (int i = 0; i < npre; i++) {
                    load_a(ks, i);
                    advance(t, ks);
                }
            } else {
                for (int i = 0; i < npre; i++) advance(t, ks);
            }
            int issued = npre;
            for (int i = npre; i < n_units; i++) {
                const int s = i % STAGES;
                const uint32_t ph = (uint32_t)((i / STAGES) & 1);
                if (!mbar_wait_bounded(empty0 + 8 * s, ph ^ 1, abort_flag, &g_gemm_error, p.budget_ns)) break;
                mbar_arrive_expect_tx(full0 + 8 * s, tx);
                load_w(t, ks, s);
                if (!FUSED) load_a(ks, s);
                advance(t, ks);
                issued = i + 1;
            }
            // wait (bounded) for the copies still in flight before leaving
            for (int i = (issued > STAGES ? issued - STAGES : 0); i < issued; i++) {
                volatile uint32_t no_abort = 0;
                mbar_wait_bounded(full0 + 8 * (i % STAGES), (uint32_t)((i / STAGES) & 1), &no_abort, &g_gemm_error, p.budget_ns);
            }
        }
        __syncwarp();
    } else if (warp == 1 || (warp >= 6 && warp < 5 + NIS)) {
        const int j = warp == 1 ? 0 : warp - 5;  // issuer index
        if (lane == 0 && j < NIS) {
            // Descriptors of stage 0: a stage, atom or K step only moves the
            // 16-byte-unit start address in the low 14 bits (shared memory
            // offsets stay below 256 KB, so the add never carries out).
            const uint64_t wdesc0 = smem_desc(smem0, 16, 1024, 2);
            const uint64_t adesc0 = smem_desc(smem0 + W_BYTES, 16, 1024, 2);
            const uint64_t sfwdesc0 = smem_desc(smem0 + W_BYTES + A_BYTES, 0, 128, 0);
            const uint64_t sfadesc0 = smem_desc(smem0 + W_BYTES + A_BYTES + SFW_BYTES, 0, 128, 0);
            int i0 = 0, ks0 = ks_first;  // first unit of the segment and its K step
            bool stop = false;
            for (int seg = 0; seg < nseg && !stop; seg++) {
                const int len = (p.nk - ks0 < n_units - i0) ? p.nk - ks0 : n_units - i0;
                const int b = seg & 1;
                const int first = i0 + ((j - i0) % NIS + NIS) % NIS;  // this issuer's first unit of the segment
                // Buffer b is free once the epilogue has drained segment seg - 2.
                // Every issuer waits, also one without units here: its commit
                // below must not count toward the barrier's previous phase.
                if (seg >= 2 &&
                    !mbar_wait_bounded(acce0 + 8 * b, (uint32_t)(((seg >> 1) - 1) & 1), abort_flag, &g_gemm_error, p.budget_ns))
                    break;
                const uint32_t acc = tmem + (uint32_t)((b % Cfg::NBUF) * NIS + j) * NB;
                for (int i = first; i < i0 + len; i += NIS) {
                    const int s = i % STAGES;
                    const uint32_t ph = (uint32_t)((i / STAGES) & 1);
                    if (!mbar_wait_bounded(full0 + 8 * s, ph, abort_flag, &g_gemm_error, p.budget_ns) ||
                        (FUSED && !mbar_wait_bounded(aready0 + 8 * s, ph, abort_flag, &g_gemm_error, p.budget_ns))) {
                        stop = true;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t so = (uint64_t)((s * STAGE_BYTES) >> 4);
                    const uint32_t tsfw = tmem + Cfg::SF_COL0 + s * SF_STAGE_COLS;
                    const uint32_t tsfa = tsfw + 16;
#pragma unroll
                    for (int a = 0; a < KA; a++) {
                        tc_cp_scale_atom(tsfw + 4 * a, sfwdesc0 + so + 32 * a);
                        tc_cp_scale_atom(tsfa + 4 * a, sfadesc0 + so + 32 * a);
                    }
#pragma unroll
                    for (int kk = 0; kk < 4; kk++) {
                        const uint64_t wd = wdesc0 + so + 2 * kk;
                        const uint64_t ad = adesc0 + so + 2 * kk;
                        const int atom = (FMT == FP4_MXFP4) ? (kk >> 1) : kk;
                        const uint32_t sfid = (FMT == FP4_MXFP4) ? (uint32_t)((kk & 1) * 2) : 0u;
                        const uint32_t idesc = idesc_blockscaled(BMW, NB, FMT == FP4_MXFP4 || p.sf_e8m0, sfid, sfid);
                        tc_mma_blockscaled<FMT>(acc, wd, ad, idesc, (tsfw + 4 * atom) | (sfid << 30),
                                                (tsfa + 4 * atom) | (sfid << 30), (i == first && kk == 0) ? 0u : 1u);
                    }
                    tc_commit(empty0 + 8 * s);
                }
                if (stop) break;
                // this issuer's part of the segment is complete (at once if it had none)
                tc_commit(accf0 + 8 * b);
                i0 += len;
                ks0 = 0;
            }
            // arrives once every MMA issued above has completed
            tc_commit(drainb);
        }
        __syncwarp();
    } else {
    // ---------------- warps 2-5 (and 9-12 when fused) ----------------
    grid_dep_wait();
    float sg = 1.0f;  // the activations' NVFP4 tensor scale (fused)
    if (FUSED) {
        grid_dep_launch();
        const int qw = quantizer_index(warp, NIS);
        if (QFMT == FP4_NVFP4 && (RES || !p.gA)) {
            // One pass over x before any encoding: max |H_k x| for a computed
            // s_g (of the FP4 stream with the residual lane) and, with the
            // lane, each row's largest residual.  Whole tiles cover all of K,
            // and so does every CTA of a cluster split while x is small; with
            // amax_exchange the CTAs of a cluster split each take their K
            // slice and combine the tensor maxima through distributed shared
            // memory, whose slices cover K.  A row exponent is per CTA: its
            // partial is scaled before the cluster adds them.
            const int K32 = p.K / 32;
            const bool slice = p.csize > 1 && (RES || amax_exchange);
            const int j0 = slice ? ks_first * 8 : 0;
            const int j1 = slice ? min((ks_first + n_units) * 8, K32) : K32;
            float mx = act_amax<HK, RES, Cfg::NQ>(p, j0, j1, qw, lane, s_red, s_rowmax);
            if (p.gA) {
                sg = *p.gA;
            } else {
                if (amax_exchange) {
                    if (qw == 0 && lane < p.csize) {
                        const uint32_t rk = cluster_ctarank();
                        st_shared_cluster_f32(mapa_shared(smem_u32(&s_amax[rk]), (uint32_t)lane), mx);
                        mbar_arrive_remote_release(mapa_shared(amaxb, (uint32_t)lane));
                    }
                    mbar_wait_cluster_bounded(amaxb, 0, abort_flag, &g_gemm_error, p.budget_ns);
                    mx = 0.0f;
                    for (int r = 0; r < p.csize; r++) mx = fmaxf(mx, s_amax[r]);
                }
                sg = nv_global_from_amax(mx);
            }
            if (RES && qw == 0 && lane < BNA) s_rexp[lane] = residual_row_exponent(__uint_as_float(s_rowmax[lane]));
            quantizers_sync<Cfg::NQ>();  // s_rexp
        } else if (QFMT == FP4_NVFP4) {
            sg = *p.gA;
        }
        if (warp == 2 && lane == 0) s_sg = sg;
        // NVFP4: the block scales' decode and encode factors for this s_g, once
        // per CTA (the quantize kernels' tables: the same values as computing
        // each factor per block, without a reciprocal per block)
        if (QFMT == FP4_NVFP4) {
            nv_tables_fill(s_tab, sg, qw * 32 + lane, Cfg::NQ * 32);
            quantizers_sync<Cfg::NQ>();
        }
        quantize_act_stages<QFMT, HK, RES, Cfg>(p, smem, aready0, empty0, n_units, t_first, ks_first, qw, lane, sg,
                                                s_rexp, QFMT == FP4_NVFP4 ? &s_tab : nullptr, abort_flag);
    }
    if (!FUSED || warp <= 5) {  // the four warps after the issuers only quantize
    // ---------------- epilogue warps 2-5: one result per tile segment ----------------
    // warp w may only read TMEM lanes 32*(w%4) .. 32*(w%4)+31
    const int quarter = warp & 3;
    const float alpha = (FMT == FP4_NVFP4 && !p.sf_e8m0) ? __fmul_rn(FUSED ? sg : *p.gA, *p.gW) : 1.0f;
    for (int seg = 0; seg < nseg; seg++) {
        const int b = seg & 1;
        const bool ok = !*abort_flag && mbar_wait_bounded(accf0 + 8 * b, (uint32_t)((seg >> 1) & 1), abort_flag,
                                                          &g_gemm_error, p.budget_ns);
        if (!epilogue_all(ok)) break;
        tc_fence_after();
        // the segment's units and the issuers that own some of them
        const int i0 = seg == 0 ? 0 : (p.nk - ks_first) + (seg - 1) * p.nk;
        const int len = (seg == 0) ? ((p.nk - ks_first < n_units) ? p.nk - ks_first : n_units)
                                   : ((p.nk < n_units - i0) ? p.nk : n_units - i0);
        uint32_t r[16];
        const uint32_t lanes = (uint32_t)(quarter * 32) << 16;
        // sum: the activations' accumulators; rsum / rsum1: the residual
        // lane's term rows (NVFP4: bands 0 and 1)
        float sum[BNA], rsum[BNA], rsum1[BNA];
#pragma unroll
        for (int m = 0; m < BNA; m++) sum[m] = rsum[m] = rsum1[m] = 0.0f;
#pragma unroll
        for (int j = 0; j < NIS; j++) {
            if (((j - i0) % NIS + NIS) % NIS >= len) continue;  // issuer j owns no unit of this segment
            const uint32_t accj = tmem + (uint32_t)((b % Cfg::NBUF) * NIS + j) * NB + lanes;
            tmem_ld16(accj, r);
            tmem_ld_wait();
#pragma unroll
            for (int m = 0; m < BNA; m++) sum[m] = __fadd_rn(sum[m], __uint_as_float(r[m]));
#pragma unroll
            for (int d = 1; d <= ND; d++) {
                tmem_ld16(accj + BNA * d, r);
                tmem_ld_wait();
                float *dst = (QFMT == FP4_NVFP4 && d > 2) ? rsum1 : rsum;
#pragma unroll
                for (int m = 0; m < BNA; m++) dst[m] = __fadd_rn(dst[m], __uint_as_float(r[m]));
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(acce0 + 8 * b) : "memory");
        // the residual sums of NVFP4 rows: back to the row's scale, band by band
        if (RES && QFMT == FP4_NVFP4) {
#pragma unroll
            for (int m = 0; m < BNA; m++)
                rsum[m] = __fadd_rn(__fmul_rn(rsum[m], exp2i(s_rexp[m])),
                                    __fmul_rn(rsum1[m], exp2i(s_rexp[m] - RES_BAND_SHIFT)));
        }
        const int t = t_first + seg;
        const int row = quarter * 32 + lane;  // row of the W tile = output column n
        const int n = t * BMW + row;
        if (p.csize > 1) {
            // cluster split (one segment per CTA): leave the partial for the
            // cluster's first CTA
#pragma unroll
            for (int q = 0; q < 4; q++) {
                part[q * 128 + row] = make_float4(sum[4 * q], sum[4 * q + 1], sum[4 * q + 2], sum[4 * q + 3]);
                if (RES)
                    part[512 + q * 128 + row] = make_float4(rsum[4 * q], rsum[4 * q + 1], rsum[4 * q + 2], rsum[4 * q + 3]);
            }
            continue;
        }
        const int c_lo = unit_owner((int64_t)t * p.nk, U, p.G), c_hi = unit_owner((int64_t)(t + 1) * p.nk - 1, U, p.G);
        if (FUSED || c_lo == c_hi) {
            // the whole K range of this tile is ours (the fused kernels run
            // whole-tile and cluster splits only): store C directly
            float acc[BNA];
#pragma unroll
            for (int m = 0; m < BNA; m++) acc[m] = __fadd_rn(0.0f, sum[m]);
            if (n < p.N) {
                if (RES) {
                    float aR[BNA];
                    const float gw = (FMT == FP4_NVFP4 && !p.sf_e8m0) ? *p.gW : 1.0f;
#pragma unroll
                    for (int m = 0; m < BNA; m++) aR[m] = gw;
                    store_row_res(p, n, acc, rsum, alpha, aR);
                } else {
                    store_row(p, n, acc, alpha);
                }
            }
            continue;
        }
        float4 *dst = reinterpret_cast<float4 *>(p.ws + (((int64_t)c * p.maxseg + seg) * 128 + row) * 16);
#pragma unroll
        for (int q = 0; q < 4; q++) dst[q] = make_float4(sum[4 * q], sum[4 * q + 1], sum[4 * q + 2], sum[4 * q + 3]);
        if (p.counters) {
            // Fused reduction: the last of the tile's c_hi - c_lo + 1 CTAs to get
            // here sums every partial in CTA order (the same order as
            // reduce_kernel, so results do not depend on which CTA is last).
            __threadfence();
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (threadIdx.x == 64) s_last = (atomicAdd(&p.counters[t], 1u) == (unsigned)(c_hi - c_lo)) ? 1u : 0u;
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (s_last) {
                __threadfence();
                float acc[BNA];
#pragma unroll
                for (int m = 0; m < BNA; m++) acc[m] = 0.0f;
                for (int cc = c_lo; cc <= c_hi; cc++) {
                    const int sg2 = t - (int)(unit_begin(cc, U, p.G) / p.nk);
                    const float4 *src = reinterpret_cast<const float4 *>(p.ws + (((int64_t)cc * p.maxseg + sg2) * 128 + row) * 16);
#pragma unroll
                    for (int q = 0; q < 4; q++) {
                        const float4 v = __ldcg(src + q);
                        acc[4 * q] = __fadd_rn(acc[4 * q], v.x);
                        acc[4 * q + 1] = __fadd_rn(acc[4 * q + 1], v.y);
                        acc[4 * q + 2] = __fadd_rn(acc[4 * q + 2], v.z);
                        acc[4 * q + 3] = __fadd_rn(acc[4 * q + 3], v.w);
                    }
                }
                if (n < p.N) store_row(p, n, acc, alpha);
                if (threadIdx.x == 64) p.counters[t] = 0u;  // ready for the next call
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");  // s_last is reused by the next segment
        }
    }
    }
    }
    tc_fence_before();
    __syncthreads();
    if (p.csize > 1) {
        // Every partial of the cluster is in place once all its CTAs pass
        // this barrier; the first CTA sums them in rank order (the CTA order
        // of the global reduction) and stores C.  The second barrier keeps
        // the other CTAs' shared memory alive until it has read it.  Both are
        // reached on every path, the abort paths included.
        cluster_sync();
        if (cluster_ctarank() == 0 && warp >= 2 && warp <= 5) {
            const int row = (warp & 3) * 32 + lane;
            const int t = c / p.csize;
            const int n = t * BMW + row;
            float acc[BNA], racc[BNA];
#pragma unroll
            for (int m = 0; m < BNA; m++) acc[m] = racc[m] = 0.0f;
            for (int rk = 0; rk < p.csize; rk++) {
#pragma unroll
                for (int q = 0; q < 4; q++) {
                    const float4 v = ld_shared_cluster_f32x4(mapa_shared(smem_u32(part + q * 128 + row), (uint32_t)rk));
                    acc[4 * q] = __fadd_rn(acc[4 * q], v.x);
                    acc[4 * q + 1] = __fadd_rn(acc[4 * q + 1], v.y);
                    acc[4 * q + 2] = __fadd_rn(acc[4 * q + 2], v.z);
                    acc[4 * q + 3] = __fadd_rn(acc[4 * q + 3], v.w);
                    if (RES) {
                        const float4 u = ld_shared_cluster_f32x4(mapa_shared(smem_u32(part + 512 + q * 128 + row), (uint32_t)rk));
                        racc[4 * q] = __fadd_rn(racc[4 * q], u.x);
                        racc[4 * q + 1] = __fadd_rn(racc[4 * q + 1], u.y);
                        racc[4 * q + 2] = __fadd_rn(racc[4 * q + 2], u.z);
                        racc[4 * q + 3] = __fadd_rn(racc[4 * q + 3], u.w);
                    }
                }
            }
            const bool nv = FMT == FP4_NVFP4 && !p.sf_e8m0;
            const float sgA = FUSED ? s_sg : (nv ? *p.gA : 1.0f);
            if (n < p.N && !*abort_flag) {
                const float alpha = nv ? __fmul_rn(sgA, *p.gW) : 1.0f;
                if (RES) {
                    float aR[BNA];
                    const float gw = nv ? *p.gW : 1.0f;
#pragma unroll
                    for (int m = 0; m < BNA; m++) aR[m] = gw;
                    store_row_res(p, n, acc, racc, alpha, aR);
                } else {
                    store_row(p, n, acc, alpha);
                }
            }
        }
        cluster_sync();
    }
    if (warp == 1) {
        tc_fence_after();
        // every MMA has completed before TMEM is released (also on the abort path)
        volatile uint32_t no_abort = 0;
        mbar_wait_bounded(drainb, 0, &no_abort, &g_gemm_error, p.budget_ns);
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// C[m][n] = alpha * sum over the CTAs that own a part of n's tile, in CTA
// order, for the tiles cut between CTAs (whole tiles were stored directly).
template <int FMT>
__global__ void __launch_bounds__(128) reduce_kernel(Params p)
{
    grid_dep_wait();
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    if (n >= p.N) return;
    const float alpha = (FMT == FP4_NVFP4 && !p.sf_e8m0) ? __fmul_rn(*p.gA, *p.gW) : 1.0f;
    const int t = n / BMW, r = n % BMW;
    const int64_t U = (int64_t)p.ntiles * p.nk;
    const int c_lo = unit_owner((int64_t)t * p.nk, U, p.G), c_hi = unit_owner((int64_t)(t + 1) * p.nk - 1, U, p.G);
    if (c_lo == c_hi) return;
    float acc[BNA];
#pragma unroll
    for (int m = 0; m < BNA; m++) acc[m] = 0.0f;
    for (int c = c_lo; c <= c_hi; c++) {
        const int seg = t - (int)(unit_begin(c, U, p.G) / p.nk);
        const float4 *src = reinterpret_cast<const float4 *>(p.ws + (((int64_t)c * p.maxseg + seg) * 128 + r) * 16);
#pragma unroll
        for (int q = 0; q < 4; q++) {
            const float4 v = src[q];
            acc[4 * q] = __fadd_rn(acc[4 * q], v.x);
            acc[4 * q + 1] = __fadd_rn(acc[4 * q + 1], v.y);
            acc[4 * q + 2] = __fadd_rn(acc[4 * q + 2], v.z);
            acc[4 * q + 3] = __fadd_rn(acc[4 * q + 3], v.w);
        }
    }
    store_row(p, n, acc, alpha);
}

struct Plan {
    int G, maxseg, nk, ntiles;
    int csize;       // cluster split: CTAs per tile (1: not a cluster split)
    bool any_cut;    // some tile is cut between CTAs outside a cluster (global reduction)
    size_t ws_bytes;
};

// Work split (see the comment above the kernel):
//   ntiles > SMs          stream-K: G = SMs CTAs over the units;
//   ntiles <= SMs / 16    global split: S = min(SMs / ntiles, nk) slices per tile;
//   otherwise             S = the largest power of two <= 8 with ntiles * S
//                         <= SMs (and S <= nk); S > 1 is a cluster split.
inline Plan plan(int64_t M, int64_t N, int64_t K, int sms)
{
    Plan pl;
    pl.nk = (int)((K + BK - 1) / BK);
    pl.ntiles = (int)((N + BMW - 1) / BMW);
    pl.csize = 1;
    const int64_t U = (int64_t)pl.ntiles * pl.nk;
    if (pl.ntiles > sms) {
        pl.G = (int)(U < sms ? U : sms);
    } else if ((int64_t)pl.ntiles * 2 * MAX_CLUSTER <= sms) {
        int64_t split = sms / pl.ntiles;
        if (split > pl.nk) split = pl.nk;
        pl.G = (int)(pl.ntiles * split);
    } else {
        int split = 1;
        while (split * 2 <= MAX_CLUSTER && (int64_t)pl.ntiles * split * 2 <= sms && split * 2 <= pl.nk) split *= 2;
        pl.G = pl.ntiles * split;
        pl.csize = split;
    }
    pl.maxseg = 1;
    for (int c = 0; c < pl.G; c++) {
        const int64_t a = unit_begin(c, U, pl.G), b = unit_begin(c + 1, U, pl.G);
        const int segs = (int)((b - 1) / pl.nk - a / pl.nk + 1);
        if (segs > pl.maxseg) pl.maxseg = segs;
    }
    pl.any_cut = false;
    if (pl.csize == 1)
        for (int t = 0; t < pl.ntiles && !pl.any_cut; t++)
            pl.any_cut = unit_owner((int64_t)t * pl.nk, U, pl.G) != unit_owner((int64_t)(t + 1) * pl.nk - 1, U, pl.G);
    pl.ws_bytes = pl.any_cut ? (size_t)pl.G * pl.maxseg * 128 * BNA * sizeof(float) : 0;
    (void)M;
    return pl;
}

// A split without tiles cut between CTAs outside a cluster, one tile segment
// per CTA (the residual variant's): plan()'s whole tiles or cluster split;
// instead of its global split, clusters of up to MAX_CLUSTER slices for few
// tiles, or one CTA per tile, in several waves, for more tiles than SMs.
inline Plan plan_nocut(int64_t M, int64_t N, int64_t K, int sms)
{
    Plan pl = plan(M, N, K, sms);
    if (!pl.any_cut && pl.maxseg == 1) return pl;
    if (pl.ntiles > sms) {
        pl.G = pl.ntiles;
        pl.csize = 1;
    } else {
        int split = 1;
        while (split * 2 <= MAX_CLUSTER && (int64_t)pl.ntiles * split * 2 <= sms && split * 2 <= pl.nk) split *= 2;
        pl.G = pl.ntiles * split;
        pl.csize = split;
    }
    pl.maxseg = 1;
    pl.any_cut = false;
    pl.ws_bytes = 0;
    return pl;
}

}  // namespace decode

// ---------------------------------------------------------------------------
// Host side
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// Row-major packed fp4 matrix (rows x K/2 bytes) as a 2-D byte tensor, boxes
// of 128 bytes x box_rows rows with 128-byte swizzle; out-of-range rows read 0.
static bool make_fp4_map(CUtensorMap *m, const void *base, int64_t rows, int64_t K, int box_rows)
{
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
    cuuint32_t box[2] = {128u, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}


// Scale-atom buffer (tile layout) as a 3-D tensor: 512-byte atoms (256
// uint16), nkb4 atoms per 128-row block, nrb row blocks; boxes of
// `box_atoms` consecutive atoms of one row block.  Atoms past a row block's
// nkb4 (a K tail) or past the last row block read as zeros.
static bool make_sf_map(CUtensorMap *m, const void *base, int64_t nkb4, int64_t nrb, int box_atoms)
{
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {256u, (cuuint64_t)nkb4, (cuuint64_t)nrb};
    cuuint64_t strides[2] = {512u, (cuuint64_t)(nkb4 * 512)};
    cuuint32_t box[3] = {256u, (cuuint32_t)box_atoms, 1u};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Raises a kernel's dynamic shared-memory limit on the current device.  The
// attribute belongs to the device's context, so it is set once per (kernel,
// device) pair; the set of pairs done is guarded for calls from several host
// threads.
static cudaError_t set_smem_limit(const void *kern, int bytes)
{
    static std::mutex mu;
    static std::set<std::pair<const void *, int>> done;
    int dev = 0;
    if (cudaError_t e = cudaGetDevice(&dev); e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    if (done.count({kern, dev})) return cudaSuccess;
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done.insert({kern, dev});
    return e;
}

template <int FMT, int OUT, int CG>
static cudaError_t launch_pgemm(const uint8_t *Aq, const uint8_t *As, const uint8_t *Wq, const uint8_t *Ws,
                                const PParams &p, int sms, cudaStream_t st, bool pdl)
{
    using Cfg = PCfg<CG>;
    constexpr int KA = (FMT == FP4_MXFP4) ? 2 : 4;
    CUtensorMap ta, tb, tsa, tsb;
    const int64_t nrb_a = (int64_t)((p.M + 127) / 128), nrb_w = (int64_t)((p.N + 127) / 128);
    if (!make_fp4_map(&ta, Aq, p.M, p.K, Cfg::BM) || !make_fp4_map(&tb, Wq, p.N, p.K, Cfg::B_ROWS) ||
        !make_sf_map(&tsa, As, p.nkb4, nrb_a, KA) || !make_sf_map(&tsb, Ws, p.nkb4, nrb_w, KA))
        return cudaErrorInvalidValue;
    auto kern = pgemm_kernel<FMT, OUT, CG>;
    if (cudaError_t e = set_smem_limit(reinterpret_cast<const void *>(kern), Cfg::SMEM_BYTES); e != cudaSuccess)
        return e;
    const int tiles = p.num_m_tiles * p.num_n_tiles;
    const int groups = tiles < sms / CG ? tiles : sms / CG;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(groups * CG, 1, 1);
    cfg.blockDim = dim3(Cfg::THREADS, 1, 1);
    cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CG;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 2 : 1;
    count_launches(1);
    return cudaLaunchKernelEx(&cfg, kern, ta, tb, tsa, tsb, p);
}

template <int FMT, int CG>
static cudaError_t launch_pgemm_out(int out, const uint8_t *Aq, const uint8_t *As, const uint8_t *Wq, const uint8_t *Ws,
                                    const PParams &p, int sms, cudaStream_t st, bool pdl)
{
    switch (out) {
    case OUT_F32: return launch_pgemm<FMT, OUT_F32, CG>(Aq, As, Wq, Ws, p, sms, st, pdl);
    case OUT_BF16: return launch_pgemm<FMT, OUT_BF16, CG>(Aq, As, Wq, Ws, p, sms, st, pdl);
    case OUT_MXFP4: return launch_pgemm<FMT, OUT_MXFP4, CG>(Aq, As, Wq, Ws, p, sms, st, pdl);
    case OUT_NVFP4: return launch_pgemm<FMT, OUT_NVFP4, CG>(Aq, As, Wq, Ws, p, sms, st, pdl);
    }
    return cudaErrorInvalidValue;
}

template <int CG>
static cudaError_t launch_pgemm_fmt(int fmt, int out, const uint8_t *Aq, const uint8_t *As, const uint8_t *Wq,
                                    const uint8_t *Ws, const PParams &p, int sms, cudaStream_t st, bool pdl)
{
    return fmt == FP4_MXFP4 ? launch_pgemm_out<FP4_MXFP4, CG>(out, Aq, As, Wq, Ws, p, sms, st, pdl)
                            : launch_pgemm_out<FP4_NVFP4, CG>(out, Aq, As, Wq, Ws, p, sms, st, pdl);
}

// CTA-pair (2-SM MMA) tiles are used once A spans more than one 128-row block.
static int pgemm_cta_group(int64_t M) { return M > 128 ? 2 : 1; }

constexpr int64_t kDecodeMaxM = 16;

// Failure-detection test hook (fp4_test_inject_stall): consumed by the next
// GEMM launch.
static std::atomic<int> g_inject_stall{0};
static std::atomic<uint64_t> g_inject_budget{0};
constexpr uint64_t kWaitBudgetNs = 2000000000ull;

size_t gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, int, int sms)
{
    if (M < 1 || M > kDecodeMaxM || N < 1 || K < 32) return 0;
    return decode::plan(M, N, K, sms).ws_bytes;
}

template <int QFMT, int HK, bool FUSED, bool RES = false>
static cudaError_t launch_decode(const CUtensorMap &tw, const CUtensorMap &ta, const CUtensorMap &tsw,
                                 const CUtensorMap &tsa, const decode::Params &p, bool any_cut, cudaStream_t st, bool pdl)
{
    constexpr int FMT = QFMT == FP4_MXFP4 ? FP4_MXFP4 : FP4_NVFP4;
    constexpr int smem = RES ? decode::DRes<QFMT>::SMEM_BYTES : decode::DPlain::SMEM_BYTES;
    auto kern = decode::decode_kernel<QFMT, HK, FUSED, RES>;
    if (cudaError_t e = set_smem_limit(reinterpret_cast<const void *>(kern), smem); e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.G);
    using Cfg = typename std::conditional<RES, decode::DRes<QFMT>, decode::DPlain>::type;
    cfg.blockDim = dim3(decode::decode_threads(FUSED, Cfg::NIS, Cfg::NQ - 4));
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (p.csize > 1) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = p.csize;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        na++;
    }
    if (pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        na++;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    count_launches(1);
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, tw, ta, tsw, tsa, p);
    if (e != cudaSuccess || FUSED || p.counters || !any_cut) return e;
    // the reduction waits for the split-K kernel inside (grid_dep_wait)
    return launch_k(decode::reduce_kernel<FMT>, dim3((p.N + 127) / 128), dim3(128), 0, st, true, p);
}

cudaError_t launch_gemm(const uint8_t *Aq, const uint8_t *As, const float *gA, const uint8_t *Wq, const uint8_t *Ws,
                        const float *gW, int64_t M, int64_t N, int64_t K, int fmt, int bf16out, void *C, int64_t ldc,
                        void *ws, size_t ws_bytes, int sms, cudaStream_t st, int *bad, bool pdl, unsigned *counters,
                        bool w_before_wait)
{
    if (M > (1 << 30) || N > (1 << 30) || K > (1 << 30)) {
        *bad = 1;
        return cudaSuccess;
    }
    const int stall = g_inject_stall.exchange(0);
    uint64_t budget = g_inject_budget.exchange(0);
    if (budget == 0) budget = kWaitBudgetNs;
    if (M <= kDecodeMaxM) {
        const decode::Plan pl = decode::plan(M, N, K, sms);
        if (pl.ws_bytes > 0 && (!ws || ws_bytes < pl.ws_bytes)) {
            *bad = 1;
            return cudaSuccess;
        }
        const int64_t nkb4 = (K / (fmt == FP4_MXFP4 ? 32 : 16) + 3) / 4;
        const int KA = fmt == FP4_MXFP4 ? 2 : 4;
        CUtensorMap tw, ta, tsw, tsa;
        if (!make_fp4_map(&tw, Wq, N, K, decode::BMW) || !make_fp4_map(&ta, Aq, M, K, decode::BNA) ||
            !make_sf_map(&tsw, Ws, nkb4, (N + 127) / 128, KA) || !make_sf_map(&tsa, As, nkb4, 1, KA))
            return cudaErrorInvalidValue;
        decode::Params dp;
        dp.ws = static_cast<float *>(ws);
        dp.N = (int)N;
        dp.M = (int)M;
        dp.K = (int)K;
        dp.nk = pl.nk;
        dp.ntiles = pl.ntiles;
        dp.G = pl.G;
        dp.maxseg = pl.maxseg;
        dp.csize = pl.csize;
        dp.w_before_wait = (pdl && w_before_wait) ? 1 : 0;
        dp.counters = counters;
        dp.budget_ns = budget;
        dp.stall = stall;
        dp.gA = gA;
        dp.gW = gW;
        dp.C = C;
        dp.ldc = ldc;
        dp.bf16out = bf16out;
        dp.sf_e8m0 = fmt == FP4_MXFP4_16;
        dp.x = nullptr;
        dp.ldx = 0;
        dp.xwide = 0;
        dp.ck = 1.0f;
        dp.round_away = dp.mx_floor = 0;
        return fmt == FP4_MXFP4 ? launch_decode<FP4_MXFP4, 0, false>(tw, ta, tsw, tsa, dp, pl.any_cut, st, pdl)
                                : launch_decode<FP4_NVFP4, 0, false>(tw, ta, tsw, tsa, dp, pl.any_cut, st, pdl);
    }
    {
        PParams pp;
        pp.gA = gA;
        pp.gW = gW;
        pp.C = C;
        pp.ldc = ldc;
        pp.Cs = nullptr;
        pp.gC = nullptr;
        pp.nkb4c = 0;
        pp.round_away = pp.mx_floor = 0;
        pp.M = (int)M;
        pp.N = (int)N;
        pp.K = (int)K;
        pp.nkb4 = (int)((K / (fmt == FP4_MXFP4 ? 32 : 16) + 3) / 4);
        pp.sf_e8m0 = fmt == FP4_MXFP4_16;
        pp.budget_ns = budget;
        pp.stall = stall;
        const int cg = pgemm_cta_group(M);
        pp.num_m_tiles = (int)((M + 128 * cg - 1) / (128 * cg));
        pp.num_n_tiles = (int)((N + 255) / 256);
        const int out = bf16out ? OUT_BF16 : OUT_F32;
        return cg == 2 ? launch_pgemm_fmt<2>(fmt, out, Aq, As, Wq, Ws, pp, sms, st, pdl)
                       : launch_pgemm_fmt<1>(fmt, out, Aq, As, Wq, Ws, pp, sms, st, pdl);
    }
}

// C = A W^T quantized along N by the prefill kernel's epilogue (M > 16,
// K % 32 == 0, N % 128 == 0; checked by the caller).
cudaError_t launch_gemm_quantized(const uint8_t *Aq, const uint8_t *As, const float *gA, const uint8_t *Wq,
                                  const uint8_t *Ws, const float *gW, int64_t M, int64_t N, int64_t K, int fmt,
                                  int out_fmt, int round_away, int mx_floor, const float *gC, uint8_t *Cq, uint8_t *Cs,
                                  int sms, cudaStream_t st)
{
    PParams pp;
    pp.gA = gA;
    pp.gW = gW;
    pp.C = Cq;
    pp.ldc = N / 2;
    pp.Cs = Cs;
    pp.gC = gC;
    pp.nkb4c = (int)((N / (out_fmt == FP4_MXFP4 ? 32 : 16) + 3) / 4);
    pp.round_away = round_away;
    pp.mx_floor = mx_floor;
    pp.M = (int)M;
    pp.N = (int)N;
    pp.K = (int)K;
    pp.nkb4 = (int)((K / (fmt == FP4_MXFP4 ? 32 : 16) + 3) / 4);
    pp.sf_e8m0 = fmt == FP4_MXFP4_16;
    uint64_t budget = g_inject_budget.exchange(0);
    pp.budget_ns = budget ? budget : kWaitBudgetNs;
    pp.stall = g_inject_stall.exchange(0);
    const int cg = pgemm_cta_group(M);
    pp.num_m_tiles = (int)((M + 128 * cg - 1) / (128 * cg));
    pp.num_n_tiles = (int)((N + 255) / 256);
    const int out = out_fmt == FP4_MXFP4 ? OUT_MXFP4 : OUT_NVFP4;
    return cg == 2 ? launch_pgemm_fmt<2>(fmt, out, Aq, As, Wq, Ws, pp, sms, st, true)
                   : launch_pgemm_fmt<1>(fmt, out, Aq, As, Wq, Ws, pp, sms, st, true);
}

template <int QFMT, bool RES>
static cudaError_t launch_linear_fused_k(int hk, const CUtensorMap &tw, const CUtensorMap &tsw, const decode::Params &p,
                                         cudaStream_t st)
{
    switch (hk) {
    case 0: return launch_decode<QFMT, 0, true, RES>(tw, tw, tsw, tsw, p, false, st, true);
    case 16: return launch_decode<QFMT, 16, true, RES>(tw, tw, tsw, tsw, p, false, st, true);
    case 32: return launch_decode<QFMT, 32, true, RES>(tw, tw, tsw, tsw, p, false, st, true);
    case 64: return launch_decode<QFMT, 64, true, RES>(tw, tw, tsw, tsw, p, false, st, true);
    case 128: return launch_decode<QFMT, 128, true, RES>(tw, tw, tsw, tsw, p, false, st, true);
    }
    return cudaErrorInvalidValue;
}

// fp4_linear for M <= 16 in one launch: the decode kernel quantizes the bf16
// activations itself (decode_kernel<..., FUSED>).  Work splits that cut a
// tile between CTAs outside a cluster (very few tiles, or stream-K) are left
// to the two-launch path: *taken = false, nothing launched.  With `residual`
// (fp4_linear_residual) the sparse residual lane is added to the product and
// every shape is taken.
cudaError_t launch_linear_fused(const uint16_t *x, int64_t ldx, int64_t M, int64_t K, int fmt, int hk, float ck,
                                int round_away, int mx_floor, const float *gA, const uint8_t *Wq, const uint8_t *Ws,
                                const float *gW, int64_t N, int bf16out, void *C, int64_t ldc, int sms, cudaStream_t st,
                                bool w_before_wait, bool residual, bool *taken)
{
    *taken = false;
    if (M < 1 || M > kDecodeMaxM || N < 1 || K < 32 || N > (1 << 30) || K > (1 << 30)) return cudaSuccess;
    // fp4_linear keeps the two-launch path for splits that cut tiles; the
    // residual lane takes a split without cuts for every shape
    const decode::Plan pl = residual ? decode::plan_nocut(M, N, K, sms) : decode::plan(M, N, K, sms);
    if (pl.any_cut) return cudaSuccess;
    *taken = true;
    const int stall = g_inject_stall.exchange(0);
    uint64_t budget = g_inject_budget.exchange(0);
    if (budget == 0) budget = kWaitBudgetNs;
    const int64_t nkb4 = (K / (fmt == FP4_MXFP4 ? 32 : 16) + 3) / 4;
    const int KA = fmt == FP4_MXFP4 ? 2 : 4;
    CUtensorMap tw, tsw;
    if (!make_fp4_map(&tw, Wq, N, K, decode::BMW) || !make_sf_map(&tsw, Ws, nkb4, (N + 127) / 128, KA))
        return cudaErrorInvalidValue;
    decode::Params dp;
    dp.ws = nullptr;
    dp.counters = nullptr;
    dp.N = (int)N;
    dp.M = (int)M;
    dp.K = (int)K;
    dp.nk = pl.nk;
    dp.ntiles = pl.ntiles;
    dp.G = pl.G;
    dp.maxseg = pl.maxseg;
    dp.csize = pl.csize;
    dp.w_before_wait = w_before_wait ? 1 : 0;
    dp.budget_ns = budget;
    dp.stall = stall;
    dp.gA = fmt == FP4_NVFP4 ? gA : nullptr;
    dp.gW = gW;
    dp.C = C;
    dp.ldc = ldc;
    dp.bf16out = bf16out;
    dp.sf_e8m0 = fmt == FP4_MXFP4_16;
    dp.x = x;
    dp.ldx = ldx;
    dp.xwide = ((reinterpret_cast<uintptr_t>(x) & 31) == 0 && (ldx * 2) % 32 == 0) ? 1 : 0;
    dp.ck = ck;
    dp.round_away = round_away;
    dp.mx_floor = mx_floor;
    if (residual) {
        switch (fmt) {
        case FP4_MXFP4: return launch_linear_fused_k<FP4_MXFP4, true>(hk, tw, tsw, dp, st);
        case FP4_NVFP4: return launch_linear_fused_k<FP4_NVFP4, true>(hk, tw, tsw, dp, st);
        case FP4_MXFP4_16: return launch_linear_fused_k<FP4_MXFP4_16, true>(hk, tw, tsw, dp, st);
        }
        return cudaErrorInvalidValue;
    }
    switch (fmt) {
    case FP4_MXFP4: return launch_linear_fused_k<FP4_MXFP4, false>(hk, tw, tsw, dp, st);
    case FP4_NVFP4: return launch_linear_fused_k<FP4_NVFP4, false>(hk, tw, tsw, dp, st);
    case FP4_MXFP4_16: return launch_linear_fused_k<FP4_MXFP4_16, false>(hk, tw, tsw, dp, st);
    }
    return cudaErrorInvalidValue;
}

cudaError_t read_and_clear_device_errors(cudaStream_t st, unsigned int *err)
{
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return e;
    unsigned int v = 0;
    if ((e = cudaMemcpyFromSymbol(&v, g_gemm_error, sizeof v)) != cudaSuccess) return e;
    const unsigned int zero = 0;
    if ((e = cudaMemcpyToSymbol(g_gemm_error, &zero, sizeof zero)) != cudaSuccess) return e;
    *err = v;
    return cudaSuccess;
}

}  // namespace fp4

namespace fp4 {

// ---------------------------------------------------------------------------
// Allocation-free decode GEMM.
//
// Some callers cannot allocate device memory at the point where they run the
// decode product: code executing inside a CUDA stream capture that must not
// add allocation nodes, plugins handed fixed buffers by a host framework, or
// processes whose memory budget is fixed up front.  For them the decode
// kernel's split-K partials live in a fixed, statically sized device array
// owned by this library instead of a caller workspace.  The array is a
// file-scope __device__ variable, so every GPU that loads the library keeps
// it (kNoAllocScratchBytes) until the process exits.
namespace {
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;  // 4 MiB
constexpr int kMaxDevices = 64;
}  // namespace

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch array on the current device.  Host code only
// sees a host-side stand-in under the array's name, so the address is looked
// up once per device (with that device current) and cached.
static cudaError_t noalloc_scratch(int dev, void **out)
{
    static std::mutex mu;
    static void *ptrs[kMaxDevices] = {};
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!ptrs[dev]) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        ptrs[dev] = p;
    }
    *out = ptrs[dev];
    return cudaSuccess;
}

}  // namespace fp4

extern "C" fp4_status fp4_test_inject_stall(int stall, uint64_t budget_ns)
{
    fp4::g_inject_budget.store(budget_ns);
    fp4::g_inject_stall.store(stall ? 1 : 0);
    return FP4_OK;
}

extern "C" fp4_status fp4_gemm_decode_noalloc(const uint8_t *Aq, const uint8_t *As, const float *gA,
                                              const uint8_t *Wq, const uint8_t *Ws, const float *gW,
                                              int64_t M, int64_t N, int64_t K, int fmt, int out_dtype,
                                              void *C, int64_t ldc, void *stream)
{
    if (M < 0 || N < 0 || K < 0 || ldc < N) return FP4_ERR_INVALID_ARG;
    if (fmt != FP4_MXFP4 && fmt != FP4_NVFP4 && fmt != FP4_MXFP4_16) return FP4_ERR_UNSUPPORTED;
    if (out_dtype != FP4_OUT_F32 && out_dtype != FP4_OUT_BF16) return FP4_ERR_INVALID_ARG;
    if (K % 32 || M > fp4::kDecodeMaxM) return FP4_ERR_UNSUPPORTED;
    if (M == 0 || N == 0) return FP4_OK;
    if (!Aq || !As || !Wq || !Ws || !C) return FP4_ERR_INVALID_ARG;
    if (fmt == FP4_NVFP4 && (!gA || !gW)) return FP4_ERR_INVALID_ARG;
    auto aligned16 = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
    if (!aligned16(Aq) || !aligned16(Wq) || !aligned16(As) || !aligned16(Ws) || !aligned16(C))
        return FP4_ERR_ALIGNMENT;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
        return FP4_ERR_CUDA;
    if (fp4::gemm_workspace_bytes(M, N, K, fmt, sms) > fp4::kNoAllocScratchBytes) return FP4_ERR_UNSUPPORTED;
    void *scratch = nullptr;
    if (fp4::noalloc_scratch(dev, &scratch) != cudaSuccess) return FP4_ERR_CUDA;
    int bad = 0;
    const cudaError_t e = fp4::launch_gemm(Aq, As, gA, Wq, Ws, gW, M, N, K, fmt, out_dtype == FP4_OUT_BF16, C, ldc,
                                           scratch, fp4::kNoAllocScratchBytes, sms,
                                           static_cast<cudaStream_t>(stream), &bad, false, nullptr, false);
    if (bad) return FP4_ERR_UNSUPPORTED;
    return e == cudaSuccess ? FP4_OK : FP4_ERR_CUDA;
}
