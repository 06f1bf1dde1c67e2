// attend_sm100.cu -- bf16 tensor-core attention over the selected cluster
// blocks plus centroid compensation of every skipped key cluster, in one
// online softmax, on tcgen05 / TMEM (sm_100a).
//
// Method: "SVG-EAR measured error" (frontier-cs.org blog), toy example: a
// skipped cluster of n keys with centroid score s_bar weighs n e^{s_bar} and
// carries its mean value; SVG-EAR task page (agent step 3): the skipped
// cluster is one key at its centroid, its score raised by log n, and every
// row returns to its place; SVG2 summary, section 3.4: permutation validity
// and the dynamic block-size kernel, which loads exactly the selected tokens
// through a per-token address table and computes dense MMAs on them.
//
// B200 design: warps 8 and 9 fill the K and V rings by TMA (a key tile is the
// next 128 entries of the query cluster's compacted list of selected key
// rows, each contiguous run copied as 2-D boxes of 2^h rows; after the key
// tiles the skipped clusters' bf16 centroids are gathered row by row), warp 10
// issues every tcgen05.mma, and two softmax warpgroups (one row per thread,
// TMEM lane = row) turn S into bf16 P in TMEM, which the PV MMA reads as its A
// operand.  O is rescaled in TMEM only when a row's running max grows by more
// than 2^8, and the epilogue writes O[q_perm[p]].  Two kernels:
//   * attend_sm100_kernel (without the variance term): one CTA per 128-row
//     tile; the softmax warpgroups take the two 64-key halves of every key
//     tile with separate softmax states and accumulators, merged at the end,
//     and S is double-buffered so QK of the next tile overlaps the softmax;
//   * attend_pair_sm100_kernel (with the variance term): one CTA per pair of
//     128-row tiles sharing every key tile, one softmax warpgroup per tile,
//     the MMAs of one tile running while the other's softmax works.
// Every wait is bounded (tc_wait.cuh); on expiry the CTA records
// SVGEAR_ERR_TIMEOUT in the device status word, drains and returns, and every
// later wait of the launch gives up at once.
#include <math.h>

#include "common.cuh"
#include "launchers.h"
#include "tc_ptx.cuh"
#include "tc_wait.cuh"
#include "tma_host.h"

namespace svgear {
namespace sm100 {

using bf16 = __nv_bfloat16;
using tc::wait_bar;
using tc::warp_wait_bar;

constexpr int BM = 128;                // query rows per half
constexpr int BN = 128;                // keys per tile
constexpr int KSTAGES = 2;             // K ring (a third stage measured no faster)
constexpr int VSTAGES = 2;             // V ring
constexpr int kHalves = 2;             // query halves per CTA
constexpr int kSoftmaxThreads = 128;   // per half: one row each
constexpr int kKWarp = 8;              // K ring producer
constexpr int kVWarp = 9;              // V ring producer
constexpr int kMmaWarp = 10;           // issues every MMA, owns the TMEM allocation
constexpr int kThreads = 12 * 32;      // 168 registers per thread at launch
// Register split: the softmax warpgroups (0-1) grow to kSoftmaxRegs, the
// producer/MMA warpgroup (2) shrinks to kIssueRegs.  The CTA's pool is
// kThreads x (registers at launch); the host refuses a build whose launch
// count is below kMinLaunchRegs, under which the split would not fit.
constexpr uint32_t kSoftmaxRegs = 232;
constexpr uint32_t kIssueRegs = 40;
constexpr int kMinLaunchRegs =
    (int)((2 * 128 * kSoftmaxRegs + 128 * kIssueRegs + kThreads - 1) / kThreads + 7) / 8 * 8;
static_assert(kMinLaunchRegs <= 168, "register split exceeds the launch allocation");
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;   // log2 units

// Tensor maps of one launch: K and V rows as 2-D boxes of 2^h rows (h = 0..7,
// for the contiguous runs of a gathered tile), the bf16 centroid tables read a
// row at a time (tile::gather4), and the query rows as 128-row boxes.
struct TmaMaps {
    CUtensorMap k[8];
    CUtensorMap v[8];
    CUtensorMap kb;
    CUtensorMap vb;
    CUtensorMap k2b;   // bf16 lambda*scale/2 * key variance, read a row at a time
    CUtensorMap q;
};

struct Shared {
    uint64_t q_full;
    uint64_t k_full[KSTAGES];
    uint64_t k_empty[KSTAGES];
    uint64_t v_full[VSTAGES];
    uint64_t v_empty[VSTAGES];
    uint64_t s_full[kHalves];
    uint64_t p_full[kHalves];
    uint64_t q2_full[kHalves];   // q^2 of the half in TMEM (variance term, no exact tiles)
    uint64_t o_full;
    uint32_t tmem_base;
    int abort_flag;
    int keep_tmem;
};

__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}
__device__ __forceinline__ uint64_t pack2(float lo, float hi) {
    return (uint64_t)__float_as_uint(lo) | ((uint64_t)__float_as_uint(hi) << 32);
}
// (o0, o1) = (x0, x1) * m + a on packed fp32 pairs
__device__ __forceinline__ void fma2(uint32_t x0, uint32_t x1, uint64_t m, uint64_t a, uint32_t& o0,
                                     uint32_t& o1) {
    asm("{\n\t.reg .b64 x, r;\n\tmov.b64 x, {%2, %3};\n\t"
        "fma.rn.f32x2 r, x, %4, %5;\n\tmov.b64 {%0, %1}, r;\n\t}"
        : "=r"(o0), "=r"(o1) : "r"(x0), "r"(x1), "l"(m), "l"(a));
}
// s += (p0, p1) on a packed fp32 pair
__device__ __forceinline__ void add2(uint64_t& s, float p0, float p1) {
    asm("{\n\t.reg .b64 x;\n\tmov.b64 x, {%1, %2};\n\tadd.rn.f32x2 %0, %0, x;\n\t}"
        : "+l"(s) : "f"(p0), "f"(p1));
}

// Swizzled 16-byte chunk address inside a tile of 128 rows x (regions of
// 64 bf16): region g covers elements [64g, 64g+64) of every row.
__device__ __forceinline__ uint32_t swz(uint32_t tile, int row, int chunk) {
    const int region = chunk >> 3, cc = chunk & 7;
    return tile + region * 16384 + row * 128 + ((cc ^ (row & 7)) << 4);
}

// q^2 of this thread's query row (read from the 128B-swizzled Q tile in
// shared memory) as bf16 pairs -- dimension 2c in the low half of column c --
// into the D/2 TMEM columns at taddr: the A operand of the variance MMA.
template <int D>
__device__ __forceinline__ void write_q2(uint32_t sQh, int r, uint32_t taddr) {
#pragma unroll
    for (int half = 0; half < D / 64; ++half) {
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            uint32_t w[4];
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                         : "r"(swz(sQh, r, half * 8 + c)));
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float lo = __uint_as_float(w[e] << 16), hi = __uint_as_float(w[e] & 0xFFFF0000u);
                __nv_bfloat162 q2 = __floats2bfloat162_rn(lo * lo, hi * hi);
                pk[4 * c + e] = *reinterpret_cast<uint32_t*>(&q2);
            }
        }
        tc::tmem_st32(taddr + half * 32, pk);
    }
}


// Producer of the K (isK) or V ring of one CTA, run by a whole warp; lane 0
// arrives on the barriers.  Tile j goes to slot j % NS once the slot's
// previous tile is released.  A key tile is the next 128 entries of the query
// cluster's list of selected keys, a concatenation of contiguous key-cluster
// segments: every run [g, g+n) of rows that falls in the tile is copied with
// 2-D boxes of 2^h rows (the binary digits of n), landing 128B-swizzled at its
// place in the tile.  Tile rows past the list are boxes at an out-of-range row
// (zeros).  Compensation tiles gather the skipped clusters' bf16 centroids row
// by row (CW clusters a tile: 128, or 64 with the variance term).
template <int D>
__device__ __forceinline__ void produce_ring(const TmaMaps& maps, bool isK, int lane,
                                             uint64_t* ring_full, uint64_t* ring_empty,
                                             uint32_t ring0, int NS, int T, int T_real, int L,
                                             int CW, int use_var, int ncomp, int nseg,
                                             const int32_t* __restrict__ pre,
                                             const int32_t* __restrict__ srow,
                                             const int32_t* __restrict__ cidx, int krow0, int kend,
                                             int crow0, int cend, volatile int* abort_flag,
                                             int* err) {
    constexpr int REG = D / 64;
    constexpr uint32_t kTileBytes = REG * 16384;
    const CUtensorMap* mrows = isK ? maps.k : maps.v;
    const CUtensorMap* mcent = isK ? &maps.kb : &maps.vb;
    int seg = 0;
    for (int j = 0; j < T; ++j) {
        const int st = j % NS;
        if (j >= NS &&
            !warp_wait_bar(&ring_empty[st], ((j / NS) - 1) & 1, abort_flag, err, (1 << 16) + j))
            break;
        const uint32_t bar = tc::smem_u32(&ring_full[st]);
        const uint32_t tX = ring0 + st * kTileBytes;
        if (j >= T_real) {
            // compensation tile: lane i gathers tile rows 4i..4i+3.  With the
            // variance term a tile covers 64 clusters: K rows 0-63 are their
            // centroids and rows 64-127 the same clusters' variance rows; V rows
            // 64-127 are zeros (read past the table)
            const int sub = use_var ? (lane & 15) : lane;
            const CUtensorMap* src = (use_var && isK && lane >= 16) ? &maps.k2b : mcent;
            int y[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int p = (j - T_real) * CW + 4 * sub + k;
                y[k] = (p < ncomp && (isK || !use_var || lane < 16)) ? crow0 + cidx[p] : cend;
            }
            if (lane == 0) tc::mbar_arrive_expect_tx(bar, BN * D * 2);
            __syncwarp();
#pragma unroll 1
            for (int g = 0; g < REG; ++g)
                tc::tma_gather4(tX + g * 16384 + lane * 512, src, g * 64, y[0], y[1], y[2], y[3],
                                bar);
        } else {
            // Lane i copies the run of segment seg + i that falls in the tile
            // (a window of 32 segments: the bounds and first rows come in with
            // two coalesced loads; a tile that spans more segments takes
            // further windows), and lane 0 zero-fills the rows past the list.
            // A run of n rows is covered by at most two boxes of 2^k rows,
            // k = floor(log2 n): one at its start and one ending at its end;
            // where they overlap both write the same bytes.  Each lane adds
            // its boxes' bytes to the barrier's expected count before issuing
            // them, and lane 0 arrives once every lane has done so.
            const int t0 = j * BN, t1 = t0 + BN, tend = min(t1, L);
            auto issue_run = [&](int r, int g, int n) {   // tile rows [r, r+n) <- rows [g, g+n)
                const int k = 31 - __clz(n), h2 = 1 << k;
                tc::mbar_expect_tx(bar, (n == h2 ? 1u : 2u) * (uint32_t)h2 * (uint32_t)(D * 2));
#pragma unroll 1
                for (int gg = 0; gg < REG; ++gg)
                    tc::tma_load_2d(tX + gg * 16384 + r * 128, &mrows[k], gg * 64, g, bar);
                if (n != h2) {
                    const int r2 = r + n - h2, g2 = (g == kend) ? kend : g + n - h2;
#pragma unroll 1
                    for (int gg = 0; gg < REG; ++gg)
                        tc::tma_load_2d(tX + gg * 16384 + r2 * 128, &mrows[k], gg * 64, g2, bar);
                }
            };
            int s0 = seg;
            unsigned done_mask;
            for (;;) {
                const int s = s0 + lane;
                int a = L, b = L;
                if (s < nseg) {
                    a = __ldg(pre + s);
                    b = __ldg(pre + s + 1);
                }
                const int lo = max(a, t0), hi = min(b, tend);
                if (lo < hi) issue_run(lo - t0, krow0 + __ldg(srow + s) + (lo - a), hi - lo);
                // segments of the window that end by t1: the next tile starts
                // in the first one that does not
                done_mask = __ballot_sync(0xffffffffu, s < nseg && b <= t1);
                const int last_end = __shfl_sync(0xffffffffu, b, 31);
                if (last_end >= tend || s0 + 32 >= nseg) break;
                s0 += 32;
            }
            seg = s0 + __popc(done_mask);
            if (lane == 0 && tend < t1) issue_run(tend - t0, kend, t1 - tend);   // zeros
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(bar);
        }
        __syncwarp();
    }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
attend_pair_sm100_kernel(const __grid_constant__ TmaMaps maps, int Nq, int Nk, int Cq, int Ck,
                         int BH, const int32_t* __restrict__ q_perm, const int4* __restrict__ tiles,
                         const int32_t* __restrict__ ntiles, int maxT,
                         const int4* __restrict__ meta, const int32_t* __restrict__ seg_prefix,
                         const int32_t* __restrict__ seg_row, const int32_t* __restrict__ comp_idx,
                         const float* __restrict__ comp_bias, float scale_log2, int use_var,
                         bf16* __restrict__ O, int* __restrict__ err, int* __restrict__ lost) {
    constexpr int REG = D / 64;                 // 64-element regions per row
    constexpr uint32_t kTileBytes = REG * 16384;
    const int bh = blockIdx.y;
    if ((int)blockIdx.x >= ntiles[bh]) return;
    // an earlier CTA already gave up, or the device's TMEM was lost before
    if (tc::refuse_start(lost, err)) return;
    const int4 tile = tiles[(size_t)bh * maxT + blockIdx.x];
    const int ci = tile.x, q0 = tile.y, q_end = tile.z;
    const int nh = (q0 + BM < q_end) ? 2 : 1;     // query halves with rows
    const int4 mt = meta[(size_t)bh * Cq + ci];   // {nseg, L keys, ncomp, 0}
    const int nseg = mt.x, L = mt.y, ncomp = mt.z;
    const int T_real = (L + BN - 1) / BN;
    // compensation tiles take CW skipped clusters: 128, or 64 with the
    // variance term (the upper 64 columns of S_h then hold q^2 of the half)
    const int CW = use_var ? BN / 2 : BN;
    const int T = T_real + (ncomp + CW - 1) / CW;

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ Shared sh;
    const uint32_t base = (tc::smem_u32(smem_raw) + 1023u) & ~1023u;
    const uint32_t sQ0 = base;                          // kHalves query tiles
    const uint32_t sK0 = sQ0 + kHalves * kTileBytes;
    const uint32_t sV0 = sK0 + KSTAGES * kTileBytes;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        tc::mbar_init(tc::smem_u32(&sh.q_full), 1);
        for (int s = 0; s < KSTAGES; ++s) {
            tc::mbar_init(tc::smem_u32(&sh.k_full[s]), 1);
            tc::mbar_init(tc::smem_u32(&sh.k_empty[s]), 1);
        }
        for (int s = 0; s < VSTAGES; ++s) {
            tc::mbar_init(tc::smem_u32(&sh.v_full[s]), 1);
            tc::mbar_init(tc::smem_u32(&sh.v_empty[s]), 1);
        }
        for (int h = 0; h < kHalves; ++h) {
            tc::mbar_init(tc::smem_u32(&sh.s_full[h]), 1);
            tc::mbar_init(tc::smem_u32(&sh.p_full[h]), kSoftmaxThreads);
            tc::mbar_init(tc::smem_u32(&sh.q2_full[h]), kSoftmaxThreads);
        }
        tc::mbar_init(tc::smem_u32(&sh.o_full), 1);
        sh.abort_flag = 0;
        sh.keep_tmem = 0;
        tc::mbar_init_fence();
    }
    if (warp == kMmaWarp) {
        tc::tmem_alloc(tc::smem_u32(&sh.tmem_base), kTmemCols);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = sh.tmem_base;
    volatile int* abort_flag = &sh.abort_flag;

    const size_t head = (size_t)bh * Nq * D;
    const size_t row_meta = ((size_t)bh * Cq + ci) * Ck;

    if (warp >= 4 * kHalves) {
    // ================================================ warpgroup 2: TMA and MMA
    tc::regs_dec<kIssueRegs>();   // one call site for the whole warpgroup
    if (warp == kKWarp || warp == kVWarp) {
        // ------------------------------------------------------------ producers
        // Warp 8 fills the K ring (a slot is freed once the QK of every half
        // that reads it is done), warp 9 the V ring (likewise with PV).
        const bool isK = warp == kKWarp;
        uint64_t* ring_full = isK ? sh.k_full : sh.v_full;
        uint64_t* ring_empty = isK ? sh.k_empty : sh.v_empty;
        const uint32_t ring0 = isK ? sK0 : sV0;
        if (isK && lane == 0) {
            tc::prefetch_tmap(&maps.q);
            const uint32_t qb = tc::smem_u32(&sh.q_full);
            tc::mbar_arrive_expect_tx(qb, nh * BM * D * 2);
            for (int h = 0; h < nh; ++h)
#pragma unroll
                for (int g = 0; g < REG; ++g)
                    tc::tma_load_2d(sQ0 + h * kTileBytes + g * 16384, &maps.q, g * 64,
                                    bh * Nq + q0 + h * BM, qb);
        }
        const int32_t* pre = seg_prefix + ((size_t)bh * Cq + ci) * (Ck + 1);
        produce_ring<D>(maps, isK, lane, ring_full, ring_empty, ring0, isK ? KSTAGES : VSTAGES, T, T_real,
                        L, CW, use_var, ncomp, nseg, pre, seg_row + row_meta, comp_idx + row_meta,
                        bh * Nk, BH * Nk, bh * Ck, BH * Ck, abort_flag, err);
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issue
        // Lane 0 runs the loop alone (MMA, commit and fence are single-thread
        // operations; the warp meets again after the drain), so nothing in the
        // loop makes it wait for the tensor core to take its queued MMAs.
        // Step j issues, per half h: PV_h(j-1) once P_h(j-1) is in TMEM, then
        // QK_h(j) into S_h (over P_h(j-1): MMAs of one thread run in order).
        // While half 0's softmax works on S_0(j), the tensor pipe runs
        // PV_1(j-1) and QK_1(j), and the other way round; the fixed order keeps
        // the two softmax warpgroups half a step apart, so they do not contend
        // for the exp unit at the same time.
        constexpr uint32_t kIdescQK = tc::idesc_bf16(BM, BN, false);
        constexpr uint32_t kIdescQK64 = tc::idesc_bf16(BM, BN / 2, false);
        constexpr uint32_t kIdescPV = tc::idesc_bf16(BM, D, true);
        if (lane == 0) {
        bool ok_run = wait_bar(&sh.q_full, 0, abort_flag, err, (5 << 16));
        for (int j = 0; ok_run && j <= T; ++j) {
            const int st = j % KSTAGES, pst = (j + VSTAGES - 1) % VSTAGES;
            for (int h = 0; h < nh; ++h) {
                if (j > 0) {
                    if ((h == 0 && !wait_bar(&sh.v_full[pst], ((j - 1) / VSTAGES) & 1, abort_flag, err,
                                             (11 << 16) + j)) ||
                        !wait_bar(&sh.p_full[h], (j - 1) & 1, abort_flag, err, (8 << 16) + (h << 12) + j)) {
                        ok_run = false;
                        break;
                    }
                    tc::fence_after_sync();
                    const uint32_t tV = sV0 + pst * kTileBytes;
                    const int kdepth = (j - 1 >= T_real) ? CW : BN;   // keys of tile j-1
                    if (kdepth == BN) {
                        tc::mma_bf16_ts_k128(tmem + kHalves * BN + h * D, tmem + h * BN,
                                             tc::sw128_desc(tV, 16384, 1024), kIdescPV, j > 1 ? 1u : 0u);
                    } else {
#pragma unroll 1
                        for (int ks = 0; ks < kdepth / 16; ++ks)
                            tc::mma_bf16_ts(tmem + kHalves * BN + h * D, tmem + h * BN + ks * 8,
                                            tc::sw128_desc(tV + ks * 2048, 16384, 1024), kIdescPV,
                                            (j > 1 || ks > 0) ? 1u : 0u);
                    }
                }
                if (j < T) {
                    if (h == 0 && !wait_bar(&sh.k_full[st], (j / KSTAGES) & 1, abort_flag, err, (6 << 16) + j)) {
                        ok_run = false;
                        break;
                    }
                    const bool var_tile = use_var && j >= T_real;
                    // q^2 of the half must be in TMEM: written with P(T_real-1), or,
                    // with no exact tiles, before the first compensation tile
                    if (var_tile && j == 0) {
                        if (!wait_bar(&sh.q2_full[h], 0, abort_flag, err, (12 << 16) + h)) {
                            ok_run = false;
                            break;
                        }
                        tc::fence_after_sync();
                    }
                    const uint32_t tQ = sQ0 + h * kTileBytes, tK = sK0 + st * kTileBytes;
                    if (D == 128 && !var_tile) {
                        tc::mma_bf16_k128(tmem + h * BN, tc::sw128_desc(tQ, 16, 1024),
                                          tc::sw128_desc(tK, 16, 1024), kIdescQK, 0u);
                    } else {
#pragma unroll 1
                        for (int ks = 0; ks < D / 16; ++ks) {
                            const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
                            tc::mma_bf16(tmem + h * BN, tc::sw128_desc(tQ + off, 16, 1024),
                                         tc::sw128_desc(tK + off, 16, 1024),
                                         var_tile ? kIdescQK64 : kIdescQK, ks > 0);
                        }
                    }
                    if (var_tile) {
                        // S += q^2 . (lambda*scale/2 Var)^T: A = q^2 from TMEM
                        // (columns 64-127 of S_h), B = tile rows 64-127
#pragma unroll 1
                        for (int ks = 0; ks < D / 16; ++ks) {
                            const uint32_t off = (ks >> 2) * 16384 + 64 * 128 + (ks & 3) * 32;
                            tc::mma_bf16_ts(tmem + h * BN, tmem + h * BN + BN / 2 + ks * 8,
                                            tc::sw128_desc(tK + off, 16, 1024), kIdescQK64, 1u);
                        }
                    }
                    tc::commit(tc::smem_u32(&sh.s_full[h]));
                }
            }
            if (!ok_run) break;
            if (j < T) tc::commit(tc::smem_u32(&sh.k_empty[st]));
            if (j > 0) tc::commit(tc::smem_u32(&sh.v_empty[pst]));
        }
        tc::commit(tc::smem_u32(&sh.o_full));
        // drain: every MMA of this CTA is complete once o_full flips; if that
        // wait expires, TMEM is left allocated rather than released under a
        // running MMA, and the device's lost word makes every later CTA and
        // launch return before it allocates
        if (!wait_bar(&sh.o_full, 0, abort_flag, err, (9 << 16))) {
            sh.keep_tmem = 1;
            tc::mark_tmem_lost(lost);
        }
        }
        __syncwarp();
    }
    } else {
    // ================================================ warpgroups 0-1: softmax
    tc::regs_inc<kSoftmaxRegs>();   // one call site for both warpgroups
    {
        // ------------------------------------------------------------ softmax
        const int h = warp >> 2;                         // query half
        const int r = tid & (kSoftmaxThreads - 1);       // row in the half == TMEM lane
        const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const uint32_t sS = lane_base + h * BN;          // S_h; P_h over its first 64 columns
        const uint32_t sO = lane_base + kHalves * BN + h * D;
        const float* cb = comp_bias + row_meta;
        float m_use = -INFINITY, l = 0.f;
        bool ok_run = h < nh;
        const bool need_q2 = use_var && ncomp > 0;
        if (ok_run && need_q2) {
            // the Q tile is read from shared memory below: wait for its copy
            ok_run = warp_wait_bar(&sh.q_full, 0, abort_flag, err, (13 << 16) + h);
            if (ok_run && T_real == 0) {   // no exact tiles: q^2 goes in first
                write_q2<D>(sQ0 + h * kTileBytes, r, sS + BN / 2);
                tc::tmem_st_wait();
                tc::fence_before_sync();
                tc::mbar_arrive(tc::smem_u32(&sh.q2_full[h]));
            }
        }
        uint32_t v[BN];
        for (int j = 0; j < T && ok_run; ++j) {
            if (!warp_wait_bar(&sh.s_full[h], j & 1, abort_flag, err, (2 << 16) + j)) {
                ok_run = false;
                break;
            }
            tc::fence_after_sync();
            const bool comp = j >= T_real;
            const int valid = comp ? min(CW, ncomp - (j - T_real) * CW) : min(BN, L - j * BN);
            const float* bias = cb + (comp ? (j - T_real) * CW : 0);
            // full key tiles keep raw scores: the max scales afterwards (scale > 0)
            // and the exp pass folds the scale into its FFMA
            const bool raw = !comp && valid == BN;
            if (!raw) {
                // Compensation and partial tiles: x = s * scale * log2(e) (+ log2 n_c
                // on compensation columns), -inf past the valid columns, rewritten
                // in TMEM 32 columns at a time before the row is loaded, so this
                // rare path's registers stay out of the main one.  Chunks wholly
                // past the valid columns are left as they are (with the variance
                // term the upper half of S_h holds q^2) and masked after the load.
#pragma unroll 1
                for (int c4 = 0; c4 * 32 < valid; ++c4) {
                    uint32_t t[32];
                    tc::tmem_ld32(sS + c4 * 32, t);
                    tc::tmem_ld_wait();
                    if (comp) {
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            const int col = c4 * 32 + e;
                            t[e] = __float_as_uint(col < valid ? fmaf(__uint_as_float(t[e]), scale_log2, bias[col])
                                                               : -INFINITY);
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            const int col = c4 * 32 + e;
                            t[e] = __float_as_uint(col < valid ? __uint_as_float(t[e]) * scale_log2 : -INFINITY);
                        }
                    }
                    tc::tmem_st32(sS + c4 * 32, t);
                }
                tc::tmem_st_wait();
            }
            tc::tmem_ld32(sS + 0, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
            tc::tmem_ld32(sS + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
            tc::tmem_ld32(sS + 64, *reinterpret_cast<uint32_t(*)[32]>(&v[64]));
            tc::tmem_ld32(sS + 96, *reinterpret_cast<uint32_t(*)[32]>(&v[96]));
            tc::tmem_ld_wait();

            // S_h is in registers: with the variance term, the last exact tile
            // leaves q^2 in the upper half of S_h for the compensation tiles
            if (need_q2 && j == T_real - 1) write_q2<D>(sQ0 + h * kTileBytes, r, sS + BN / 2);
            if (!raw) {
#pragma unroll
                for (int c4 = 0; c4 < BN / 32; ++c4)
                    if (c4 * 32 >= valid)
#pragma unroll
                        for (int e = 0; e < 32; ++e) v[c4 * 32 + e] = __float_as_uint(-INFINITY);
            }
            float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
            for (int e = 0; e < BN; e += 8) {   // three-input max: half the instructions
                mx0 = fmax3(mx0, __uint_as_float(v[e]), __uint_as_float(v[e + 1]));
                mx1 = fmax3(mx1, __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
                mx2 = fmax3(mx2, __uint_as_float(v[e + 4]), __uint_as_float(v[e + 5]));
                mx3 = fmax3(mx3, __uint_as_float(v[e + 6]), __uint_as_float(v[e + 7]));
            }
            float mx = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3));
            if (raw) mx *= scale_log2;
            const float m_new = fmaxf(m_use, mx);

            // Lazy rescale of O: a row needs it when its max grew by more than
            // 2^8; the TMEM loads and stores are warp-collective, so the warp
            // rescales together when any row must (the others with alpha = 1).
            // O_h is final up to PV_h(j-1) here: that MMA was issued before
            // QK_h(j), whose commit completed s_full.
            const bool need = j > 0 && m_new > m_use + kRescaleThreshold;
            const bool any = __any_sync(0xffffffffu, need);
            float alpha = 1.f;
            if (j == 0) {
                m_use = m_new;
            } else if (need) {
                alpha = tc::ex2(m_use - m_new);
                l *= alpha;
                m_use = m_new;
            }
            // P = 2^(x - m) as bf16 pairs over the first 64 columns of S_h
            const float xs = raw ? scale_log2 : 1.f, neg_m = -m_use;
            // (even, odd) columns in packed fp32 pairs: one FFMA2 and one FADD2
            // per two scores, elementwise round-to-nearest like the scalar forms
            uint64_t s01 = 0ull;
            const uint64_t xs2 = pack2(xs, xs), nm2 = pack2(neg_m, neg_m);
#pragma unroll
            for (int q = 0; q < BN / 32; ++q) {
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    uint32_t a0, a1;
                    fma2(v[q * 32 + e], v[q * 32 + e + 1], xs2, nm2, a0, a1);
                    const float p0 = tc::ex2(__uint_as_float(a0));
                    const float p1 = tc::ex2(__uint_as_float(a1));
                    add2(s01, p0, p1);
                    __nv_bfloat162 hp = __floats2bfloat162_rn(p0, p1);
                    pk[e >> 1] = *reinterpret_cast<uint32_t*>(&hp);
                }
                tc::tmem_st16(sS + q * 16, pk);
            }
            l += __uint_as_float((uint32_t)s01) + __uint_as_float((uint32_t)(s01 >> 32));
            if (any) {
                uint32_t o[16];
#pragma unroll 1
                for (int c = 0; c < D / 16; ++c) {
                    tc::tmem_ld16(sO + c * 16, o);
                    tc::tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                    tc::tmem_st16(sO + c * 16, o);
                }
            }
            tc::tmem_st_wait();
            tc::fence_before_sync();
            tc::mbar_arrive(tc::smem_u32(&sh.p_full[h]));
        }
        // epilogue: O / l back to the original token order
        if (ok_run && T > 0 && warp_wait_bar(&sh.o_full, 0, abort_flag, err, (4 << 16))) {
            tc::fence_after_sync();
            const int p = q0 + h * BM + r;
            const float inv = 1.f / l;
            const bool write = p < q_end;
            const int dst = write ? q_perm[(size_t)bh * Nq + p] : 0;
            bf16* orow = O + head + (size_t)dst * D;
            uint32_t o[32];
#pragma unroll
            for (int c4 = 0; c4 < D / 32; ++c4) {
                tc::tmem_ld32(sO + c4 * 32, o);
                tc::tmem_ld_wait();
                if (write && (unsigned)dst < (unsigned)Nq) {
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        __nv_bfloat162 hp = __floats2bfloat162_rn(__uint_as_float(o[e]) * inv,
                                                                  __uint_as_float(o[e + 1]) * inv);
                        pk[e >> 1] = *reinterpret_cast<uint32_t*>(&hp);
                    }
                    uint4* o4 = reinterpret_cast<uint4*>(orow + c4 * 32);
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        o4[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
                }
            }
        }
    }
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == kMmaWarp && !sh.keep_tmem) tc::tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------------------
// Tile kernel: one CTA per 128-row tile of one query cluster, used without the
// variance term.  The two softmax warpgroups split every key tile by columns
// (warpgroup h takes keys [64h, 64h+64) of each tile) and keep separate online
// softmax states and output accumulators O_h, merged in the epilogue like two
// partial attentions.  S is double-buffered in TMEM, so QK of tile j+1 runs
// while the softmax works on tile j:
//   TMEM: S[0] | S[1] | O_0 | O_1 (128 + 128 + d + d columns); P of key half
//   h of tile j is written as bf16 over the first 32 columns of that half's S
//   columns in S[j % 2].
//   MMA order: QK(0), QK(1); then for every j: PV_0(j), PV_1(j) (K = 64 each,
//   O_h += P_h V[64h : 64h+64)), QK(j+2) into S[j % 2] -- MMAs of one thread
//   run in order, so QK(j+2) overwrites P(j) only after both PV read it.
// A tcgen05.mma issue returns about when the pipe can take it, so the issuing
// thread does little else: one non-blocking test of its three barriers per
// tile, one barrier for both halves' P (one arrival per softmax warp), and two
// commits per tile -- S[j % 2] full, which also frees K slot j % 2 for tile
// j+2, and V slot j % 2 empty, which also tells the softmax that both PV of
// tile j are complete (the O rescale of tile j+1 waits for it).
// ---------------------------------------------------------------------------
constexpr int KST1 = 2;   // K ring: slot j % 2, freed when QK(j) completes
constexpr int VST1 = 2;   // V ring: slot j % 2, freed when PV(j) completes

// O_0 (+)= P_0 V[0:64), O_1 (+)= P_1 V[64:128) as eight K=16 steps in one asm
// block: P_h is 32 TMEM columns at a + 64h, the V tile MN-major with its
// 16-row steps 2048 bytes (128 descriptor units) apart; step 0 of each half
// overwrites its O unless accumulate is set.
__device__ __forceinline__ void mma_pv_halves(uint32_t d0, uint32_t d1, uint32_t a, uint64_t bdesc,
                                              uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t.reg .b32 t;\n\t.reg .b64 b;\n\t"
        "setp.ne.b32 p, %5, 0;\n\t"
        "setp.ne.b32 q, %6, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%2], %3, %4, p;\n\t"
        "add.u32 t, %2, 8;\n\tadd.s64 b, %3, 128;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [t], b, %4, q;\n\t"
        "add.u32 t, %2, 16;\n\tadd.s64 b, %3, 256;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [t], b, %4, q;\n\t"
        "add.u32 t, %2, 24;\n\tadd.s64 b, %3, 384;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [t], b, %4, q;\n\t"
        "add.u32 t, %2, 64;\n\tadd.s64 b, %3, 512;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%1], [t], b, %4, p;\n\t"
        "add.u32 t, %2, 72;\n\tadd.s64 b, %3, 640;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%1], [t], b, %4, q;\n\t"
        "add.u32 t, %2, 80;\n\tadd.s64 b, %3, 768;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%1], [t], b, %4, q;\n\t"
        "add.u32 t, %2, 88;\n\tadd.s64 b, %3, 896;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%1], [t], b, %4, q;\n\t}\n" ::"r"(d0),
        "r"(d1), "r"(a), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(1u)
        : "memory");
}

struct Shared1 {
    uint64_t q_full;
    uint64_t k_full[KST1];   // (K slot j % 2 is freed by s_full[j % 2])
    uint64_t v_full[VST1];
    uint64_t v_empty[VST1];
    uint64_t s_full[2];      // S[b] holds QK of the tile j with j % 2 == b
    uint64_t p_full[2];      // [j % 2]: P of both halves of tile j in TMEM (8 warps)
    uint64_t o_full;
    uint32_t tmem_base;
    int abort_flag;
    int keep_tmem;
    float xm[2][BM];         // each key half's running max and row sum, for the merge
    float xl[2][BM];
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
attend_sm100_kernel(const __grid_constant__ TmaMaps maps, int Nq, int Nk, int Cq, int Ck, int BH,
                    const int32_t* __restrict__ q_perm, const int4* __restrict__ tiles,
                    const int32_t* __restrict__ ntiles, int maxT, const int4* __restrict__ meta,
                    const int32_t* __restrict__ seg_prefix, const int32_t* __restrict__ seg_row,
                    const int32_t* __restrict__ comp_idx, const float* __restrict__ comp_bias,
                    float scale_log2, bf16* __restrict__ O, int* __restrict__ err,
                    int* __restrict__ lost) {
    constexpr int REG = D / 64;                 // 64-element regions per row
    constexpr uint32_t kTileBytes = REG * 16384;
    constexpr int KH = BN / 2;                  // keys per softmax warpgroup and tile
    const int bh = blockIdx.y;
    if ((int)blockIdx.x >= ntiles[bh]) return;
    // an earlier CTA already gave up, or the device's TMEM was lost before
    if (tc::refuse_start(lost, err)) return;
    const int4 tile = tiles[(size_t)bh * maxT + blockIdx.x];
    const int ci = tile.x, q0 = tile.y, q_end = tile.z;
    const int4 mt = meta[(size_t)bh * Cq + ci];   // {nseg, L keys, ncomp, 0}
    const int nseg = mt.x, L = mt.y, ncomp = mt.z;
    const int T_real = (L + BN - 1) / BN;
    const int T = T_real + (ncomp + BN - 1) / BN;

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ Shared1 sh;
    const uint32_t base = (tc::smem_u32(smem_raw) + 1023u) & ~1023u;
    const uint32_t sQ = base;                           // the query tile
    const uint32_t sK0 = sQ + kTileBytes;
    const uint32_t sV0 = sK0 + KST1 * kTileBytes;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        tc::mbar_init(tc::smem_u32(&sh.q_full), 1);
        for (int s = 0; s < KST1; ++s) tc::mbar_init(tc::smem_u32(&sh.k_full[s]), 1);
        for (int s = 0; s < VST1; ++s) {
            tc::mbar_init(tc::smem_u32(&sh.v_full[s]), 1);
            tc::mbar_init(tc::smem_u32(&sh.v_empty[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            tc::mbar_init(tc::smem_u32(&sh.s_full[b]), 1);
            tc::mbar_init(tc::smem_u32(&sh.p_full[b]), 2 * kSoftmaxThreads / 32);
        }
        tc::mbar_init(tc::smem_u32(&sh.o_full), 1);
        sh.abort_flag = 0;
        sh.keep_tmem = 0;
        tc::mbar_init_fence();
    }
    if (warp == kMmaWarp) {
        tc::tmem_alloc(tc::smem_u32(&sh.tmem_base), kTmemCols);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = sh.tmem_base;
    volatile int* abort_flag = &sh.abort_flag;

    const size_t head = (size_t)bh * Nq * D;
    const size_t row_meta = ((size_t)bh * Cq + ci) * Ck;

    if (warp >= 8) {
    // ================================================ warpgroup 2: TMA and MMA
    tc::regs_dec<kIssueRegs>();   // one call site for the whole warpgroup
    if (warp == kKWarp || warp == kVWarp) {
        // Warp 8 fills the K ring (slot j % 2 is free once S[j % 2] of the
        // tile before is full), warp 9 the V ring.
        const bool isK = warp == kKWarp;
        if (isK && lane == 0) {
            tc::prefetch_tmap(&maps.q);
            const uint32_t qb = tc::smem_u32(&sh.q_full);
            tc::mbar_arrive_expect_tx(qb, BM * D * 2);
#pragma unroll
            for (int g = 0; g < REG; ++g)
                tc::tma_load_2d(sQ + g * 16384, &maps.q, g * 64, bh * Nq + q0, qb);
        }
        produce_ring<D>(maps, isK, lane, isK ? sh.k_full : sh.v_full, isK ? sh.s_full : sh.v_empty,
                        isK ? sK0 : sV0, isK ? KST1 : VST1, T, T_real, L, BN, 0, ncomp, nseg,
                        seg_prefix + ((size_t)bh * Cq + ci) * (Ck + 1), seg_row + row_meta,
                        comp_idx + row_meta, bh * Nk, BH * Nk, bh * Ck, BH * Ck, abort_flag, err);
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issue
        // Lane 0 runs the loop alone (MMA, commit and fence are single-thread
        // operations; the warp meets again after the drain).
        constexpr uint32_t kIdescQK = tc::idesc_bf16(BM, BN, false);
        constexpr uint32_t kIdescPV = tc::idesc_bf16(BM, D, true);
        if (lane == 0) {
        bool ok_run = wait_bar(&sh.q_full, 0, abort_flag, err, (5 << 16));
        // S[j % 2] = Q K(j)^T once K tile j has landed (unless the caller
        // already saw it); its commit also releases K slot j % 2
        auto issue_qk = [&](int j, bool landed) -> bool {
            const int st = j % KST1;
            if (!landed && !wait_bar(&sh.k_full[st], (j / KST1) & 1, abort_flag, err, (6 << 16) + j))
                return false;
            const uint32_t tK = sK0 + st * kTileBytes, dS = tmem + (j & 1) * BN;
            if (D == 128) {
                tc::mma_bf16_k128(dS, tc::sw128_desc(sQ, 16, 1024), tc::sw128_desc(tK, 16, 1024),
                                  kIdescQK, 0u);
            } else {
#pragma unroll 1
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
                    tc::mma_bf16(dS, tc::sw128_desc(sQ + off, 16, 1024),
                                 tc::sw128_desc(tK + off, 16, 1024), kIdescQK, ks > 0);
                }
            }
            tc::commit(tc::smem_u32(&sh.s_full[j & 1]));
            return true;
        };
        for (int j = 0; ok_run && j < T && j < 2; ++j) ok_run = issue_qk(j, false);
        for (int j = 0; ok_run && j < T; ++j) {
            const int vs = j % VST1, ks = (j + 2) % KST1;
            // V tile j, P of tile j and K tile j+2, tested together; a wait
            // only for what has not arrived
            const uint32_t m = tc::mbar_test3(tc::smem_u32(&sh.v_full[vs]), (j / VST1) & 1,
                                              tc::smem_u32(&sh.p_full[j & 1]), (j >> 1) & 1,
                                              tc::smem_u32(&sh.k_full[ks]), ((j + 2) / KST1) & 1);
            if ((!(m & 1) && !wait_bar(&sh.v_full[vs], (j / VST1) & 1, abort_flag, err, (11 << 16) + j)) ||
                (!(m & 2) && !wait_bar(&sh.p_full[j & 1], (j >> 1) & 1, abort_flag, err, (8 << 16) + j))) {
                ok_run = false;
                break;
            }
            tc::fence_after_sync();
            mma_pv_halves(tmem + 2 * BN, tmem + 2 * BN + D, tmem + (j & 1) * BN,
                          tc::sw128_desc(sV0 + vs * kTileBytes, 16384, 1024), kIdescPV, j > 0 ? 1u : 0u);
            tc::commit(tc::smem_u32(&sh.v_empty[vs]));
            if (j + 2 < T) ok_run = issue_qk(j + 2, (m & 4) != 0);
        }
        tc::commit(tc::smem_u32(&sh.o_full));
        // drain: every MMA of this CTA is complete once o_full flips; if that
        // wait expires, TMEM is left allocated rather than released under a
        // running MMA, and the device's lost word makes every later CTA and
        // launch return before it allocates
        if (!wait_bar(&sh.o_full, 0, abort_flag, err, (9 << 16))) {
            sh.keep_tmem = 1;
            tc::mark_tmem_lost(lost);
        }
        }
        __syncwarp();
    }
    } else {
    // ================================================ warpgroups 0-1: softmax
    tc::regs_inc<kSoftmaxRegs>();   // one call site for both warpgroups
    {
        const int h = warp >> 2;                         // key half of every tile
        const int r = tid & (kSoftmaxThreads - 1);       // query row == TMEM lane
        const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const uint32_t sO = lane_base + 2 * BN + h * D;
        const float* cb = comp_bias + row_meta + h * KH;
        float m_use = -INFINITY, l = 0.f;
        bool ok_run = true;
        uint32_t v[KH];
        for (int j = 0; j < T && ok_run; ++j) {
            if (!warp_wait_bar(&sh.s_full[j & 1], (j >> 1) & 1, abort_flag, err, (2 << 16) + j)) {
                ok_run = false;
                break;
            }
            tc::fence_after_sync();
            const uint32_t sS = lane_base + (j & 1) * BN + h * KH;
            const bool comp = j >= T_real;
            const int valid_all = comp ? min(BN, ncomp - (j - T_real) * BN) : min(BN, L - j * BN);
            const int valid = min(max(valid_all - h * KH, 0), KH);   // columns of this half
            const float* bias = cb + (comp ? (j - T_real) * BN : 0);
            // full key halves keep raw scores: the max scales afterwards
            // (scale > 0) and the exp pass folds the scale into its FFMA
            const bool raw = !comp && valid == KH;
            if (!raw) {
                // Compensation and partial tiles: x = s * scale * log2(e) (+ log2 n_c
                // on compensation columns), -inf past the valid columns, rewritten
                // in TMEM 32 columns at a time before the row is loaded
#pragma unroll 1
                for (int c4 = 0; c4 * 32 < valid; ++c4) {
                    uint32_t t[32];
                    tc::tmem_ld32(sS + c4 * 32, t);
                    tc::tmem_ld_wait();
                    if (comp) {
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            const int col = c4 * 32 + e;
                            t[e] = __float_as_uint(col < valid ? fmaf(__uint_as_float(t[e]), scale_log2, bias[col])
                                                               : -INFINITY);
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            const int col = c4 * 32 + e;
                            t[e] = __float_as_uint(col < valid ? __uint_as_float(t[e]) * scale_log2 : -INFINITY);
                        }
                    }
                    tc::tmem_st32(sS + c4 * 32, t);
                }
                tc::tmem_st_wait();
            }
            tc::tmem_ld32(sS + 0, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
            tc::tmem_ld32(sS + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
            tc::tmem_ld_wait();
            if (!raw) {
#pragma unroll
                for (int c4 = 0; c4 < KH / 32; ++c4)
                    if (c4 * 32 >= valid)
#pragma unroll
                        for (int e = 0; e < 32; ++e) v[c4 * 32 + e] = __float_as_uint(-INFINITY);
            }
            float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
            for (int e = 0; e < KH; e += 8) {   // three-input max: half the instructions
                mx0 = fmax3(mx0, __uint_as_float(v[e]), __uint_as_float(v[e + 1]));
                mx1 = fmax3(mx1, __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
                mx2 = fmax3(mx2, __uint_as_float(v[e + 4]), __uint_as_float(v[e + 5]));
                mx3 = fmax3(mx3, __uint_as_float(v[e + 6]), __uint_as_float(v[e + 7]));
            }
            float mx = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3));
            if (raw) mx *= scale_log2;
            const float m_new = fmaxf(m_use, mx);

            // Lazy rescale of O_h: a row needs it when its max grew by more
            // than 2^8 (or from -inf: no valid column seen yet, O_h and l are
            // zero); the TMEM loads and stores are warp-collective, so the warp
            // rescales together when any row must (the others with alpha = 1).
            const bool need = j > 0 && m_new > m_use + kRescaleThreshold;
            const bool any = __any_sync(0xffffffffu, need);
            float alpha = 1.f;
            if (j == 0) {
                m_use = m_new;
            } else if (need) {
                alpha = tc::ex2(m_use - m_new);
                l *= alpha;
                m_use = m_new;
            }
            // P = 2^(x - m) as bf16 pairs over the first 32 columns of this
            // half's S columns; a row with no valid column yet takes m = 0
            // (every x is -inf, so P = 0)
            const float xs = raw ? scale_log2 : 1.f, neg_m = m_use == -INFINITY ? 0.f : -m_use;
            uint64_t s01 = 0ull;
            const uint64_t xs2 = pack2(xs, xs), nm2 = pack2(neg_m, neg_m);
#pragma unroll
            for (int q = 0; q < KH / 32; ++q) {
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    uint32_t a0, a1;
                    fma2(v[q * 32 + e], v[q * 32 + e + 1], xs2, nm2, a0, a1);
                    const float p0 = tc::ex2(__uint_as_float(a0));
                    const float p1 = tc::ex2(__uint_as_float(a1));
                    add2(s01, p0, p1);
                    __nv_bfloat162 hp = __floats2bfloat162_rn(p0, p1);
                    pk[e >> 1] = *reinterpret_cast<uint32_t*>(&hp);
                }
                tc::tmem_st16(sS + q * 16, pk);
            }
            l += __uint_as_float((uint32_t)s01) + __uint_as_float((uint32_t)(s01 >> 32));
            if (any) {
                // O_h is final up to PV(j-1) once the commit that frees V slot
                // (j-1) % 2 completes: the rescale must not race that MMA
                if (!warp_wait_bar(&sh.v_empty[(j - 1) % VST1], ((j - 1) / VST1) & 1, abort_flag, err,
                                   (3 << 16) + j)) {
                    ok_run = false;
                    break;
                }
                tc::fence_after_sync();
                uint32_t o[16];
#pragma unroll 1
                for (int c = 0; c < D / 16; ++c) {
                    tc::tmem_ld16(sO + c * 16, o);
                    tc::tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                    tc::tmem_st16(sO + c * 16, o);
                }
            }
            tc::tmem_st_wait();
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(tc::smem_u32(&sh.p_full[j & 1]));
        }
        // Epilogue: O = (a0 O_0 + a1 O_1) / (a0 l_0 + a1 l_1), a_h = 2^(m_h - m),
        // m = max(m_0, m_1).  The two warpgroups trade (m, l) through shared
        // memory (the named barrier is reached on every path) and each writes
        // half of the row's columns, reading both partial O from its lanes.
        const bool ok = ok_run && T > 0 &&
                        warp_wait_bar(&sh.o_full, 0, abort_flag, err, (4 << 16) + h);
        sh.xm[h][r] = m_use;
        sh.xl[h][r] = l;
        asm volatile("bar.sync 1, %0;" ::"n"(2 * kSoftmaxThreads) : "memory");
        if (ok && !*abort_flag) {
            tc::fence_after_sync();
            const float m0 = sh.xm[0][r], m1 = sh.xm[1][r];
            const float mm = fmaxf(m0, m1);
            const float a0 = tc::ex2(m0 - mm), a1 = tc::ex2(m1 - mm);
            const float inv = 1.f / (a0 * sh.xl[0][r] + a1 * sh.xl[1][r]);
            const float c0 = a0 * inv, c1 = a1 * inv;
            const int p = q0 + r;
            const int dst = p < q_end ? q_perm[(size_t)bh * Nq + p] : -1;
            bf16* orow = O + head + (size_t)max(dst, 0) * D;
            const uint32_t sO0 = lane_base + 2 * BN;
            uint32_t o0[32], o1[32];
#pragma unroll
            for (int c4 = h * D / 64; c4 < (h + 1) * D / 64; ++c4) {
                tc::tmem_ld32(sO0 + c4 * 32, o0);
                tc::tmem_ld32(sO0 + D + c4 * 32, o1);
                tc::tmem_ld_wait();
                if ((unsigned)dst < (unsigned)Nq) {
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        __nv_bfloat162 hp = __floats2bfloat162_rn(
                            fmaf(__uint_as_float(o0[e]), c0, __uint_as_float(o1[e]) * c1),
                            fmaf(__uint_as_float(o0[e + 1]), c0, __uint_as_float(o1[e + 1]) * c1));
                        pk[e >> 1] = *reinterpret_cast<uint32_t*>(&hp);
                    }
                    uint4* o4 = reinterpret_cast<uint4*>(orow + c4 * 32);
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        o4[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
                }
            }
        }
    }
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == kMmaWarp && !sh.keep_tmem) tc::tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------------------
// Preparation: bf16 centroid tables, per-query-cluster key lists, tile table.
// ---------------------------------------------------------------------------
__global__ void to_bf16_kernel(const float* __restrict__ src, bf16* __restrict__ dst, size_t n,
                               float mul) {
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (size_t)gridDim.x * blockDim.x)
        dst[i] = __float2bfloat16_rn(src[i] * mul);
}

// One block per (query cluster, head).  Selected clusters in ascending order
// become segments (prefix positions, first key row); skipped non-empty
// clusters become the compensation list with bias log2(n_c).
__global__ void attend_prep_kernel(const int32_t* __restrict__ k_off, int Ck, int Cq, int Nk,
                                   const int32_t* __restrict__ pair_off,
                                   const int32_t* __restrict__ pair_kc, int4* __restrict__ meta,
                                   int32_t* __restrict__ seg_prefix, int32_t* __restrict__ seg_row,
                                   int32_t* __restrict__ comp_idx, float* __restrict__ comp_bias) {
    extern __shared__ unsigned char sel[];
    const int i = blockIdx.x, bh = blockIdx.y;
    const int32_t* ko = k_off + (size_t)bh * (Ck + 1);
    const int32_t* po = pair_off + (size_t)bh * (Cq + 1);
    const int32_t* pk = pair_kc + (size_t)bh * Cq * Ck;
    for (int c = threadIdx.x; c < Ck; c += blockDim.x) sel[c] = 0;
    __syncthreads();
    for (int e = po[i] + threadIdx.x; e < po[i + 1]; e += blockDim.x) {
        const int c = pk[e];
        if ((unsigned)c < (unsigned)Ck) sel[c] = 1;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const size_t rm = ((size_t)bh * Cq + i) * Ck;
        int32_t* pre = seg_prefix + ((size_t)bh * Cq + i) * (Ck + 1);
        int nseg = 0, L = 0, nc = 0;
        for (int c = 0; c < Ck; ++c) {
            const int a = ko[c], b = ko[c + 1];
            if (b <= a || a < 0 || b > Nk) continue;
            if (sel[c]) {
                pre[nseg] = L;
                seg_row[rm + nseg] = a;
                L += b - a;
                ++nseg;
            } else {
                comp_idx[rm + nc] = c;
                comp_bias[rm + nc] = log2f((float)(b - a));
                ++nc;
            }
        }
        pre[nseg] = L;
        for (int s = nseg + 1; s <= Ck; ++s) pre[s] = L;   // sentinels for the segment walk
        meta[(size_t)bh * Cq + i] = make_int4(nseg, L, nc, 0);
    }
}

// One block per head: every (cluster, run of `rows` query rows) of the query
// segments; a CTA takes one entry.
__global__ void attend_tiles_kernel(const int32_t* __restrict__ q_off, int Cq, int Nq, int rows,
                                    int maxT, int4* __restrict__ tiles,
                                    int32_t* __restrict__ ntiles) {
    const int bh = blockIdx.x;
    if (threadIdx.x != 0) return;
    const int32_t* qo = q_off + (size_t)bh * (Cq + 1);
    int k = 0;
    for (int i = 0; i < Cq; ++i) {
        const int a = qo[i], b = qo[i + 1];
        if (b <= a || a < 0 || b > Nq) continue;
        for (int r0 = a; r0 < b && k < maxT; r0 += rows)
            tiles[(size_t)bh * maxT + k++] = make_int4(i, r0, b, 0);
    }
    ntiles[bh] = k;
}

// The tile kernel, or the pair kernel with the variance term.  The register
// split of each needs its launch allocation, checked once per kernel.
template <int D>
int launch_attend_kernel(const TmaMaps& maps, int Nq, int Nk, int Cq, int Ck, int BH,
                         const int32_t* q_perm, const AttendWs& w, float scale_log2, int use_var,
                         bf16* O, int* lost, cudaStream_t st) {
    const void* fn = use_var ? (const void*)attend_pair_sm100_kernel<D> : (const void*)attend_sm100_kernel<D>;
    static int launch_regs[2] = {0, 0};   // [tile, pair]
    int& lr = launch_regs[use_var ? 1 : 0];
    if (lr == 0) {
        cudaFuncAttributes fa;
        if (cudaFuncGetAttributes(&fa, fn) != cudaSuccess) return SVGEAR_ERR_CUDA;
        lr = fa.numRegs;
    }
    if (lr < kMinLaunchRegs) return SVGEAR_ERR_UNSUPPORTED;
    const int tiles = use_var ? kHalves + KSTAGES + VSTAGES : 1 + KST1 + VST1;
    const size_t smem = (size_t)tiles * (D / 64) * 16384 + 1024;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return SVGEAR_ERR_CUDA;
    if (use_var)
        attend_pair_sm100_kernel<D><<<dim3(w.maxT, BH), kThreads, smem, st>>>(
            maps, Nq, Nk, Cq, Ck, BH, q_perm, w.tiles, w.ntiles, w.maxT, w.meta, w.seg_prefix,
            w.seg_row, w.comp_idx, w.comp_bias, scale_log2, use_var, O, w.status, lost);
    else
        attend_sm100_kernel<D><<<dim3(w.maxT, BH), kThreads, smem, st>>>(
            maps, Nq, Nk, Cq, Ck, BH, q_perm, w.tiles, w.ntiles, w.maxT, w.meta, w.seg_prefix,
            w.seg_row, w.comp_idx, w.comp_bias, scale_log2, O, w.status, lost);
    return SVGEAR_OK;
}

}  // namespace sm100

int launch_attend_sm100(const void* Qp, const void* Kp, const void* Vp, svgear_dims qd, int Nk,
                        const int32_t* q_off, int Cq, const int32_t* k_off, int Ck,
                        const int32_t* pair_off, const int32_t* pair_kc, const float* kbar,
                        const float* vbar, const int32_t* q_perm, float scale, void* O,
                        const float* kvar, float lambda, const AttendWs& w, cudaStream_t st) {
    using namespace sm100;
    const int BH = qd.B * qd.H;
    const int D = qd.d;
    if (tmem_lost_latched()) return SVGEAR_ERR_TMEM_LOST;
    int* lost = nullptr;
    if (int s = tmem_lost_word(&lost)) return s;
    if ((long long)BH * Nk >= (1ll << 31)) return SVGEAR_ERR_UNSUPPORTED;   // int32 TMA rows
    if ((long long)BH * qd.N >= (1ll << 31)) return SVGEAR_ERR_UNSUPPORTED;
    TmaMaps maps;
    const int use_var = (kvar != nullptr && lambda != 0.f) ? 1 : 0;
    bool ok = make_rows_map(&maps.kb, w.kbar16, (uint64_t)BH * Ck, D, 1) &&
              make_rows_map(&maps.k2b, w.k2bar16, (uint64_t)BH * Ck, D, 1) &&
              make_rows_map(&maps.vb, w.vbar16, (uint64_t)BH * Ck, D, 1) &&
              make_rows_map(&maps.q, Qp, (uint64_t)BH * qd.N, D, BM);
    for (int h = 0; h < 8 && ok; ++h)
        ok = make_rows_map(&maps.k[h], Kp, (uint64_t)BH * Nk, D, 1u << h) &&
             make_rows_map(&maps.v[h], Vp, (uint64_t)BH * Nk, D, 1u << h);
    if (!ok) return SVGEAR_ERR_CUDA;
    if (cudaMemsetAsync(w.status, 0, 4 * sizeof(int), st) != cudaSuccess) return SVGEAR_ERR_CUDA;
    const size_t nc = (size_t)BH * Ck * D;
    const int cgrid = (int)((nc + 255) / 256 < 4096 ? (nc + 255) / 256 : 4096);
    to_bf16_kernel<<<cgrid, 256, 0, st>>>(kbar, w.kbar16, nc, 1.f);
    count_launches(1);
    to_bf16_kernel<<<cgrid, 256, 0, st>>>(vbar, w.vbar16, nc, 1.f);
    count_launches(1);
    if (use_var) {
        // B operand of the variance MMA: lambda * scale / 2 * Var (the softmax
        // multiplies the raw scores by scale * log2 e)
        to_bf16_kernel<<<cgrid, 256, 0, st>>>(kvar, w.k2bar16, nc, lambda * scale * 0.5f);
        count_launches(1);
    }
    attend_prep_kernel<<<dim3(Cq, BH), 128, Ck, st>>>(k_off, Ck, Cq, Nk, pair_off, pair_kc, w.meta,
                                                      w.seg_prefix, w.seg_row, w.comp_idx,
                                                      w.comp_bias);
    count_launches(1);
    // 128-row tiles; 256-row tile pairs for the kernel with the variance term
    attend_tiles_kernel<<<BH, 32, 0, st>>>(q_off, Cq, qd.N, use_var ? kHalves * BM : BM, w.maxT,
                                           w.tiles, w.ntiles);
    count_launches(1);
    const float scale_log2 = scale * 1.4426950408889634f;
    const int s = D == 128 ? launch_attend_kernel<128>(maps, qd.N, Nk, Cq, Ck, BH, q_perm, w, scale_log2,
                                                       use_var, static_cast<bf16*>(O), lost, st)
                           : launch_attend_kernel<64>(maps, qd.N, Nk, Cq, Ck, BH, q_perm, w, scale_log2,
                                                      use_var, static_cast<bf16*>(O), lost, st);
    if (s != SVGEAR_OK) return s;
    count_launches(1);
    SVGEAR_LAUNCH_CHECK();
    return SVGEAR_OK;
}

}  // namespace svgear
