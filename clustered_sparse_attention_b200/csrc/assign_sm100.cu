// assign_sm100.cu -- k-means assignment of bf16 tokens on tcgen05 / TMEM.
//
// Method: SVG2 summary ("Sparse VideoGen2 ...", section 3.4, "The clustering
// operation"): every token joins the centroid nearest in Euclidean distance.
// argmin_c |x - c|^2 = argmin_c (|c|^2 - 2 x.c), and x.c over all tokens and
// centroids of a head is a dense contraction, which runs here on the tensor
// cores; ties keep the lowest centroid index.
//
// Precision: x is bf16, exact as an MMA operand.  Each fp32 centroid is split
// into two bf16 planes, c ~ h + m with h = bf16(c), m = bf16(c - h) (the
// difference is exact in fp32).  The residual c - h lies below half a bf16
// ulp of c, so rounding it loses at most 2^-17 |c_k| per element, and the
// split changes x.c by at most 2^-17 sum_k |x_k c_k|: the worst-case rounding
// of an fp32 dot product of length 128.  One fp32-accumulated MMA chain of
// depth 2d sums x.h + x.m, whose products are exact; for d = 128 split and
// accumulation together bound the error by the same 1.5 * 2^-16 sum_k
// |x_k c_k| as an exact three-plane split accumulated over depth 3d, for a
// third fewer MMAs and plane bytes.
//
// The norm is folded into the contraction: one more K=16 step multiplies a
// tile of ones by the centroid's -|c|^2/2 (from the fp32 centroid, split into
// three bf16 parts, which hold it to 2^-24), so the accumulator holds
// x.c - |c|^2/2 and the token's label is the column of its maximum.  The
// step adds three exact products to the fp32 chain; with the planes, the
// distance -2(x.c - |c|^2/2) errs by at most 2 (2^-17 + (2d+3) u) sum_k
// |x_k c_k| + (3d+5) u |c|^2 against |x - c|^2 - |x|^2.
//
// B200 design: persistent CTAs, one per SM, walk the 128-token tiles of all
// heads (tiles of heads at their fixed point are skipped).  Centroid planes
// stay in shared memory: all of a head's when they fit (each tile then runs
// every chunk), else one chunk's at a time, run against a group of up to
// kGroupTiles token tiles of the head before the next chunk's planes replace
// them (each token's running maximum is carried from chunk to chunk).
//   warp 0     TMA producer: the token tile (2 to 4 stages, as shared memory
//              allows) and, when the plane set changes, its boxes of Nc rows
//              x 64 dims (128B-swizzled);
//   warp 1     one lane issues tcgen05.mma (M=128, N=Nc <= 256, K=16) into one
//              of two TMEM accumulators, each centroid chunk a chain of
//              2 planes x d/16 steps;
//   warps 2-9  epilogue, two warps per TMEM lane quarter (TMEM lane = token
//              row), each scanning half of every chunk's columns for the
//              running (x.c - |c|^2/2, index) maximum; the upper half hands
//              its maximum to the lower through shared memory, which merges
//              (ties to the lower index) and writes the label.
// Every wait is bounded (tc_wait.cuh); on expiry the status word records
// SVGEAR_ERR_TIMEOUT, copies and MMAs in flight are drained and the CTA
// returns.
#include <math.h>

#include "common.cuh"
#include "launchers.h"
#include "tc_ptx.cuh"
#include "tc_wait.cuh"
#include "tma_host.h"

namespace svgear {
namespace asg {

using bf16 = __nv_bfloat16;
using tc::warp_wait_bar;

constexpr int BM = 128;                  // tokens per tile (TMEM lanes)
constexpr int kPlanes = 2;               // bf16 planes of a centroid
constexpr int kGroupTiles = 16;          // token tiles per unit when one chunk's planes are resident
constexpr int kMaxGroup = 16;            // carried minima per epilogue thread
constexpr int kThreads = 10 * 32;
constexpr int kMmaWarp = 1;
constexpr int kEpiThreads = 256;
constexpr uint32_t kTmemCols = 512;      // two accumulators of up to 256 columns
constexpr uint32_t kAccCols = 256;
constexpr int kMaxAStages = 4;           // token-tile stages: as many as shared memory holds
constexpr int kNormK = 16;               // the norm step's K: -|c|^2/2 in 3 bf16 parts, then zeros
constexpr uint32_t kOnesBytes = BM * kNormK * 2;   // the norm step's A: 128 x 16 bf16 ones
constexpr uint64_t kDrainNs = 200000000ull;    // 0.2 s to let issued work land

struct Maps {
    CUtensorMap x;   // tokens [B*H*N][D], boxes of 128 rows x 64
    CUtensorMap b;   // centroid planes [B*H][2][Cpad][D], boxes of Nc rows x 64
    CUtensorMap n;   // norm steps [B*H][Cpad][16], boxes of Nc rows x 16 (32-byte swizzle)
};

struct Shared {
    uint64_t a_full[kMaxAStages];
    uint64_t a_empty[kMaxAStages];
    uint64_t b_full;    // the current plane set is in its slots
    uint64_t b_empty;   // the MMAs of the previous plane set have completed
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t drain;
    uint64_t pair_full[4][2];    // per lane quarter and slot: the upper half's minimum is stored
    uint64_t pair_empty[4][2];   // the lower half has read it
    float pair_d[2][BM];         // the upper half's running maximum, double-buffered by tile
    uint16_t pair_i[2][BM];      // and its centroid index (C <= SVGEAR_MAX_CLUSTERS)
    uint32_t tmem_base;
    int abort_flag;
    int keep_tmem;
};

// Wait for a phase without regard to abort flags (used to let copies and MMAs
// that were issued complete before the CTA exits); false after kDrainNs.
__device__ __forceinline__ bool drain_wait(uint64_t* bar, uint32_t parity) {
    const uint32_t b = tc::smem_u32(bar);
    const uint64_t t0 = tc::global_timer_ns();
    for (uint32_t it = 0; !tc::mbar_try_wait(b, parity); ++it)
        if (tc::global_timer_ns() - t0 > kDrainNs || it >= tc::kMaxSpins) return false;
    return true;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
assign_sm100_kernel(const __grid_constant__ Maps maps, int N, int BH, int Cpad, int Nc, int nA,
                    int nB, int resident, int G, int32_t* __restrict__ labels,
                    const int32_t* __restrict__ done, int32_t* __restrict__ changed,
                    int* __restrict__ err, int* __restrict__ lost) {
    constexpr int KH = D / 64;                   // 64-dim halves of a row
    constexpr uint32_t kABytes = KH * 16384;     // 128 rows x D bf16
    // an earlier CTA already gave up, or the device's TMEM was lost before
    if (tc::refuse_start(lost, err)) return;
    const int tiles_per_head = (N + BM - 1) / BM;
    const int nchunk = Cpad / Nc;
    // Work units and plane sets.  Resident: a unit is one token tile, every
    // chunk's planes form one set per head, and each tile runs all chunks.
    // Grouped: a unit is up to G tiles of one head, a set is one chunk's
    // planes, and the unit's tiles run chunk by chunk (one phase per chunk),
    // carrying each token's running maximum from phase to phase.
    if (resident || G < 1) G = 1;
    if (G > kMaxGroup) G = kMaxGroup;
    const int units_per_head = (tiles_per_head + G - 1) / G;
    const int total = BH * units_per_head;
    const int phases = resident ? 1 : nchunk;
    const int chunks_per_step = resident ? nchunk : 1;

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ Shared sh;
    const uint32_t base = (tc::smem_u32(smem_raw) + 1023u) & ~1023u;
    const uint32_t sA0 = base;
    const uint32_t sB0 = base + nA * kABytes;
    const uint32_t kBStageBytes = (uint32_t)Nc * 128u;   // Nc rows x 64 bf16 (multiple of 2 KB)
    const uint32_t kNStageBytes = (uint32_t)Nc * 32u;    // Nc rows x 16 bf16 (multiple of 512 B)
    const uint32_t sN0 = sB0 + nB * kBStageBytes;        // norm steps of the set's chunks
    const uint32_t sOnes = sN0 + chunks_per_step * kNStageBytes;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // the norm step's A operand: bf16 ones in every element (so in any layout)
    for (uint32_t o = (uint32_t)tid * 16u; o < kOnesBytes; o += kThreads * 16u)
        asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(sOnes + o), "r"(0x3F803F80u)
                     : "memory");
    tc::fence_async_smem();   // visible to the tensor core
    if (tid == 0) {
        for (int s = 0; s < kMaxAStages; ++s) {
            tc::mbar_init(tc::smem_u32(&sh.a_full[s]), 1);
            tc::mbar_init(tc::smem_u32(&sh.a_empty[s]), 1);
        }
        for (int s = 0; s < 2; ++s) {
            tc::mbar_init(tc::smem_u32(&sh.acc_full[s]), 1);
            tc::mbar_init(tc::smem_u32(&sh.acc_empty[s]), kEpiThreads);
        }
        tc::mbar_init(tc::smem_u32(&sh.b_full), 1);
        tc::mbar_init(tc::smem_u32(&sh.b_empty), 1);
        tc::mbar_init(tc::smem_u32(&sh.drain), 1);
        for (int q = 0; q < 4; ++q)
            for (int s = 0; s < 2; ++s) {
                tc::mbar_init(tc::smem_u32(&sh.pair_full[q][s]), 32);
                tc::mbar_init(tc::smem_u32(&sh.pair_empty[q][s]), 32);
            }
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

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            tc::prefetch_tmap(&maps.x);
            tc::prefetch_tmap(&maps.b);
            tc::prefetch_tmap(&maps.n);
        }
        int ia = 0;
        int loaded = -1, hc = 0;   // plane set in the slots, plane-set changes
        bool ok = true;
        for (int u = blockIdx.x; ok && u < total; u += gridDim.x) {
            const int bh = u / units_per_head;
            if (done && done[bh]) continue;
            const int tlo = (u - bh * units_per_head) * G;
            const int thi = min(tlo + G, tiles_per_head);
            for (int ph = 0; ok && ph < phases; ++ph) {
                const int set = resident ? bh : bh * nchunk + ph;
                for (int ti = tlo; ti < thi; ++ti) {
                    const int sa = ia % nA;
                    if (ia >= nA &&
                        !warp_wait_bar(&sh.a_empty[sa], ((ia / nA) - 1) & 1, abort_flag, err, (1 << 16) + ia)) {
                        ok = false;
                        break;
                    }
                    if (lane == 0) {
                        const uint32_t bar = tc::smem_u32(&sh.a_full[sa]);
                        tc::mbar_arrive_expect_tx(bar, BM * D * 2);
#pragma unroll
                        for (int kh = 0; kh < KH; ++kh)
                            tc::tma_load_2d(sA0 + sa * kABytes + kh * 16384, &maps.x, kh * 64, bh * N + ti * BM,
                                            bar);
                    }
                    __syncwarp();
                    ++ia;
                    // the set's planes go into slots 0..nB-1 once the MMAs of the
                    // previous set have completed (after this tile's copy was issued,
                    // which the MMA warp needs before it releases the previous set)
                    if (set != loaded) {
                        if (hc > 0 &&
                            !warp_wait_bar(&sh.b_empty, (hc - 1) & 1, abort_flag, err, (2 << 16) + hc)) {
                            ok = false;
                            break;
                        }
                        if (lane == 0) {
                            const uint32_t bar = tc::smem_u32(&sh.b_full);
                            tc::mbar_arrive_expect_tx(
                                bar, (uint32_t)(nB * Nc * 128 + chunks_per_step * Nc * kNormK * 2));
                            const int c0 = resident ? 0 : ph;
                            for (int c = 0; c < chunks_per_step; ++c) {
                                for (int p = 0; p < kPlanes; ++p)
#pragma unroll
                                    for (int kh = 0; kh < KH; ++kh)
                                        tc::tma_load_2d(sB0 + ((c * kPlanes + p) * KH + kh) * kBStageBytes,
                                                        &maps.b, kh * 64,
                                                        (bh * kPlanes + p) * Cpad + (c0 + c) * Nc, bar);
                                tc::tma_load_2d(sN0 + c * kNStageBytes, &maps.n, 0, bh * Cpad + (c0 + c) * Nc,
                                                bar);
                            }
                        }
                        __syncwarp();
                        loaded = set;
                        ++hc;
                    }
                }
            }
        }
        // let the last copy into every stage land before the CTA can exit
        if (lane == 0) {
            for (int k = 0; k < nA && k < ia; ++k) {
                const int i = ia - 1 - k;
                drain_wait(&sh.a_full[i % nA], (i / nA) & 1);
            }
            if (hc > 0) drain_wait(&sh.b_full, (hc - 1) & 1);
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issue
        // Lane 0 runs the loop alone (MMA, commit and fence are single-thread
        // operations; the warp meets again after the drain), so no warp
        // barrier makes it wait for the tensor core to take its queued MMAs.
        const uint32_t idesc = tc::idesc_bf16(BM, Nc, false);
        const uint64_t ones_desc = tc::sw32_desc(sOnes, 256);
        if (lane == 0) {
        int ia = 0, ic = 0;
        int cur = -1, hc = 0;   // plane set in use, plane-set changes
        bool ok = true;
        for (int u = blockIdx.x; ok && u < total; u += gridDim.x) {
            const int bh = u / units_per_head;
            if (done && done[bh]) continue;
            const int tlo = (u - bh * units_per_head) * G;
            const int thi = min(tlo + G, tiles_per_head);
            for (int ph = 0; ok && ph < phases; ++ph) {
                const int set = resident ? bh : bh * nchunk + ph;
                for (int ti = tlo; ok && ti < thi; ++ti) {
                    const int sa = ia % nA;
                    if (!tc::wait_bar(&sh.a_full[sa], (ia / nA) & 1, abort_flag, err, (3 << 16) + ia)) {
                        ok = false;
                        break;
                    }
                    for (int c = 0; c < chunks_per_step; ++c) {
                        const int buf = ic & 1;
                        if (ic >= 2 &&
                            !tc::wait_bar(&sh.acc_empty[buf], ((ic >> 1) - 1) & 1, abort_flag, err,
                                          (4 << 16) + (ic & 0xffff))) {
                            ok = false;
                            break;
                        }
                        tc::fence_after_sync();
                        if (set != cur) {
                            // the previous set's slots are free once its MMAs
                            // complete; then wait for this set's planes
                            if (hc > 0) tc::commit(tc::smem_u32(&sh.b_empty));
                            if (!tc::wait_bar(&sh.b_full, hc & 1, abort_flag, err, (5 << 16) + hc)) {
                                ok = false;
                                break;
                            }
                            tc::fence_after_sync();
                            cur = set;
                            ++hc;
                        }
                        for (int p = 0; p < kPlanes; ++p)
                            for (int kh = 0; kh < KH; ++kh) {
                                const int sb = (c * kPlanes + p) * KH + kh;
                                const uint64_t ad0 = tc::sw128_desc(sA0 + sa * kABytes + kh * 16384, 16, 1024);
                                const uint64_t bd0 = tc::sw128_desc(sB0 + sb * kBStageBytes, 16, 1024);
#pragma unroll
                                for (int ks = 0; ks < 4; ++ks)   // +32 bytes per K=16 step
                                    tc::mma_bf16(tmem + buf * kAccCols, ad0 + 2 * ks, bd0 + 2 * ks, idesc,
                                                 (p | kh | ks) != 0 ? 1u : 0u);
                            }
                        // + ones . (-|c|^2/2 parts)
                        tc::mma_bf16(tmem + buf * kAccCols, ones_desc,
                                     tc::sw32_desc(sN0 + c * kNStageBytes, 256), idesc, 1u);
                        tc::commit(tc::smem_u32(&sh.acc_full[buf]));
                        ++ic;
                    }
                    if (!ok) break;
                    tc::commit(tc::smem_u32(&sh.a_empty[sa]));
                    ++ia;
                }
            }
        }
        // every MMA this warp issued has completed once `drain` flips; if it
        // does not, TMEM stays allocated rather than freed under a running MMA
        tc::commit(tc::smem_u32(&sh.drain));
        if (!drain_wait(&sh.drain, 0)) {
            sh.keep_tmem = 1;
            tc::mark_tmem_lost(lost);
        }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        const int quarter = warp & 3;                  // TMEM lanes this warp may read
        const int upper = (warp - 2) >> 2;             // 0: warps 2-5, 1: warps 6-9
        const int r = quarter * 32 + lane;             // token row in the tile
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        // a chunk's columns in steps of 32 (and a last step of 16 when Nc is
        // an odd multiple of 16): the lower half takes the first ceil(n/2)
        const int nfull = Nc / 32;
        const int nsteps = nfull + ((Nc & 16) ? 1 : 0);
        const int s_lo = upper ? (nsteps + 1) / 2 : 0;
        const int s_hi = upper ? nsteps : (nsteps + 1) / 2;
        int it = 0;   // tiles handed over, for the slot and its phase
        // running maximum of this thread's token in each tile of a unit,
        // carried from one phase to the next (grouped units)
        float carry_d[kMaxGroup];
        int carry_i[kMaxGroup];
        int ic = 0;
        bool ok = true;
        for (int u = blockIdx.x; ok && u < total; u += gridDim.x) {
            const int bh = u / units_per_head;
            if (done && done[bh]) continue;
            const int tlo = (u - bh * units_per_head) * G;
            const int thi = min(tlo + G, tiles_per_head);
            for (int ph = 0; ok && ph < phases; ++ph) {
                const bool last = ph == phases - 1;
                for (int ti = tlo; ok && ti < thi; ++ti) {
                    const int t = ti * BM + r;
                    int32_t* lp = labels + (size_t)bh * N + t;
                    // the previous label, loaded now and compared once the tile is done
                    const int old = (last && changed && !upper && t < N) ? *lp : -1;
                    // four interleaved running maxima of x.c - |c|^2/2 (columns e mod
                    // 4), merged with ties to the lower index: the first maximum of the
                    // sequential scan
                    float best[4];
                    int bi[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        best[e] = __int_as_float(0xff800000);
                        bi[e] = 0;
                    }
                    auto scan = [&](const uint32_t* v, int nq, int base) {
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            if (q < nq) {
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const float sc = __uint_as_float(v[4 * q + e]);
                                    if (sc > best[e]) {
                                        best[e] = sc;
                                        bi[e] = base + 4 * q + e;
                                    }
                                }
                            }
                        }
                    };
                    for (int c = 0; c < chunks_per_step; ++c) {
                        const int buf = ic & 1;
                        if (!warp_wait_bar(&sh.acc_full[buf], (ic >> 1) & 1, abort_flag, err,
                                           (6 << 16) + (ic & 0xffff))) {
                            ok = false;
                            break;
                        }
                        tc::fence_after_sync();
                        const uint32_t tb = lane_base + buf * kAccCols;
                        const int cb = (resident ? c : ph) * Nc;
                        const int hi_full = s_hi < nfull ? s_hi : nfull;   // full steps of this half
                        uint32_t va[32], vb[32];
                        // double-buffered: the next step's load is in flight while one is scanned
                        if (s_lo < hi_full) tc::tmem_ld32(tb + s_lo * 32, va);
                        for (int k = s_lo; k < hi_full; k += 2) {
                            tc::tmem_ld_wait();
                            if (k + 1 < hi_full) tc::tmem_ld32(tb + (k + 1) * 32, vb);
                            scan(va, 8, cb + k * 32);
                            if (k + 1 < hi_full) {
                                tc::tmem_ld_wait();
                                if (k + 2 < hi_full) tc::tmem_ld32(tb + (k + 2) * 32, va);
                                scan(vb, 8, cb + (k + 1) * 32);
                            }
                        }
                        if ((Nc & 16) && s_hi == nsteps && s_lo <= nfull) {   // the 16-column step
                            uint32_t v16[16];
                            tc::tmem_ld16(tb + nfull * 32, v16);
                            tc::tmem_ld_wait();
                            scan(v16, 4, cb + nfull * 32);
                        }
                        // the accumulator is in registers: the MMA may refill it
                        tc::fence_before_sync();
                        tc::mbar_arrive(tc::smem_u32(&sh.acc_empty[buf]));
                        ++ic;
                    }
                    if (!ok) break;
                    float bb = best[0];
                    int bx = bi[0];
#pragma unroll
                    for (int e = 1; e < 4; ++e)
                        if (best[e] > bb || (best[e] == bb && bi[e] < bx)) {
                            bb = best[e];
                            bx = bi[e];
                        }
                    // the upper half hands its maximum to the lower half of the same rows
                    const int slot = it & 1;
                    const uint32_t use = (uint32_t)(it >> 1);
                    ++it;
                    if (upper) {
                        if (use > 0 && !warp_wait_bar(&sh.pair_empty[quarter][slot], (use - 1) & 1, abort_flag,
                                                      err, (7 << 16) + (it & 0xffff))) {
                            ok = false;
                            break;
                        }
                        sh.pair_d[slot][r] = bb;
                        sh.pair_i[slot][r] = (uint16_t)bx;
                        tc::mbar_arrive(tc::smem_u32(&sh.pair_full[quarter][slot]));
                        continue;
                    }
                    if (!warp_wait_bar(&sh.pair_full[quarter][slot], use & 1, abort_flag, err,
                                       (8 << 16) + (it & 0xffff))) {
                        ok = false;
                        break;
                    }
                    {
                        const float ud = sh.pair_d[slot][r];
                        const int ux = sh.pair_i[slot][r];
                        tc::mbar_arrive(tc::smem_u32(&sh.pair_empty[quarter][slot]));
                        if (ud > bb || (ud == bb && ux < bx)) {
                            bb = ud;
                            bx = ux;
                        }
                    }
                    if (ph > 0) {
                        // earlier phases hold lower indices: they keep ties
                        const int g = ti - tlo;
                        if (!(bb > carry_d[g])) {
                            bb = carry_d[g];
                            bx = carry_i[g];
                        }
                    }
                    if (!last) {
                        carry_d[ti - tlo] = bb;
                        carry_i[ti - tlo] = bx;
                    } else if (t < N) {
                        if (changed && old != bx) changed[bh] = 1;
                        *lp = bx;
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

// Centroid planes and norm steps, one warp per centroid: planes[bh][p][c][k]
// for p = hi, lo, and nstep[bh][c][0..2] = -|c|^2/2 as three bf16 parts (each
// the rounding of what the previous ones leave, exact in fp32), zeros after;
// padding rows (c >= C) have zero planes and -1e30 in the norm step, so they
// never win the maximum.
template <int D>
__global__ void centroid_planes_kernel(const float* __restrict__ cent, int C, int Cpad,
                                       bf16* __restrict__ planes, bf16* __restrict__ nstep,
                                       const int32_t* __restrict__ done) {
    const int bh = blockIdx.y;
    if (done && done[bh]) return;
    const int c = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (c >= Cpad) return;
    float s = 0.f;
#pragma unroll
    for (int k = lane; k < D; k += 32) {
        const float v = c < C ? cent[((size_t)bh * C + c) * D + k] : 0.f;
        const bf16 h = __float2bfloat16_rn(v);
        const float r1 = v - __bfloat162float(h);
        const bf16 m = __float2bfloat16_rn(r1);
        const size_t row = ((size_t)bh * kPlanes * Cpad + c) * D + k;
        planes[row] = h;
        planes[row + (size_t)Cpad * D] = m;
        s = fmaf(v, v, s);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane < kNormK) {
        const float n = c < C ? -0.5f * s : -1e30f;
        const bf16 p0 = __float2bfloat16_rn(n);
        const float n1 = n - __bfloat162float(p0);
        const bf16 p1 = __float2bfloat16_rn(n1);
        const bf16 p2 = __float2bfloat16_rn(n1 - __bfloat162float(p1));
        const bf16 z = __float2bfloat16_rn(0.f);
        nstep[((size_t)bh * Cpad + c) * kNormK + lane] = lane == 0 ? p0 : lane == 1 ? p1 : lane == 2 ? p2 : z;
    }
}

// Centroid chunking: as few chunks as possible of at most 256 columns, each a
// multiple of 16 wide.
inline void chunking(int C, int* nchunk, int* Nc) {
    *nchunk = (C + 255) / 256;
    const int per = (C + *nchunk - 1) / *nchunk;
    *Nc = (per + 15) / 16 * 16;
}

}  // namespace asg

size_t assign_sm100_scratch_bytes(int BH, int C, int D) {
    int nchunk, Nc;
    asg::chunking(C, &nchunk, &Nc);
    const size_t Cpad = (size_t)nchunk * Nc;
    return (size_t)BH * Cpad * (asg::kPlanes * D + asg::kNormK) * sizeof(__nv_bfloat16);
}

int launch_assign_sm100(const void* X, svgear_dims dims, const float* cent, int C,
                        int32_t* labels, void* scratch, int* err, cudaStream_t st,
                        const int32_t* done, int32_t* changed) {
    using namespace asg;
    const int BH = dims.B * dims.H, N = dims.N, D = dims.d;
    if (tmem_lost_latched()) return SVGEAR_ERR_TMEM_LOST;
    int* lost = nullptr;
    if (int s = tmem_lost_word(&lost)) return s;
    if ((long long)BH * N >= (1ll << 31)) return SVGEAR_ERR_UNSUPPORTED;   // int32 TMA rows
    int nchunk, Nc;
    chunking(C, &nchunk, &Nc);
    const int Cpad = nchunk * Nc;
    bf16* planes = static_cast<bf16*>(scratch);
    bf16* nstep = planes + (size_t)BH * kPlanes * Cpad * D;
    Maps maps;
    if (!make_rows_map(&maps.x, X, (uint64_t)BH * N, D, BM) ||
        !make_rows_map(&maps.b, planes, (uint64_t)BH * kPlanes * Cpad, D, (uint32_t)Nc) ||
        !make_k16_map(&maps.n, nstep, (uint64_t)BH * Cpad, (uint32_t)Nc))
        return SVGEAR_ERR_CUDA;
    static int num_sms[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SVGEAR_ERR_CUDA;
    if (num_sms[dev] == 0 &&
        cudaDeviceGetAttribute(&num_sms[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return SVGEAR_ERR_CUDA;
    const int tiles = BH * ceil_div(N, BM);
    // Shared memory: the plane slots (with each chunk's norm step) and the
    // ones tile, then as many token-tile stages as fit (2 to kMaxAStages).
    // All of a head's planes stay resident when they fit beside two token
    // stages; otherwise one chunk's planes are resident per phase of a group
    // of kGroupTiles tiles.
    const size_t a_bytes = (size_t)(D / 64) * 16384, b_stage = (size_t)Nc * 128;
    const size_t n_stage = (size_t)Nc * kNormK * 2;
    // the static Shared block is placed before the 1024-aligned dynamic block
    const size_t static_bytes = (sizeof(Shared) + 1023) / 1024 * 1024;
    const size_t budget = 227 * 1024 - static_bytes - 1024;
    const int boxes_head = nchunk * kPlanes * (D / 64);
    const int resident =
        budget >= 2 * a_bytes + (size_t)boxes_head * b_stage + nchunk * n_stage + kOnesBytes ? 1 : 0;
    const int nB = resident ? boxes_head : kPlanes * (D / 64);
    const size_t b_bytes = (size_t)nB * b_stage + (resident ? nchunk : 1) * n_stage + kOnesBytes;
    if (budget < 2 * a_bytes + b_bytes) return SVGEAR_ERR_UNSUPPORTED;
    const int G = resident ? 1 : (kGroupTiles < kMaxGroup ? kGroupTiles : kMaxGroup);
    const int units = resident ? tiles : BH * ceil_div(ceil_div(N, BM), G);
    const int grid = units < num_sms[dev] ? units : num_sms[dev];
    int nA = (int)((budget - b_bytes) / a_bytes);
    if (nA > kMaxAStages) nA = kMaxAStages;
    const size_t smem = (size_t)nA * a_bytes + b_bytes + 1024;
    if (D == 128) {
        centroid_planes_kernel<128><<<dim3(ceil_div(Cpad, 8), BH), 256, 0, st>>>(cent, C, Cpad, planes,
                                                                                nstep, done);
        count_launches(1);
        if (cudaFuncSetAttribute(assign_sm100_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem) != cudaSuccess)
            return SVGEAR_ERR_CUDA;
        assign_sm100_kernel<128><<<grid, kThreads, smem, st>>>(maps, N, BH, Cpad, Nc, nA, nB, resident, G, labels,
                                                               done, changed, err, lost);
    } else {
        centroid_planes_kernel<64><<<dim3(ceil_div(Cpad, 8), BH), 256, 0, st>>>(cent, C, Cpad, planes,
                                                                               nstep, done);
        count_launches(1);
        if (cudaFuncSetAttribute(assign_sm100_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem) != cudaSuccess)
            return SVGEAR_ERR_CUDA;
        assign_sm100_kernel<64><<<grid, kThreads, smem, st>>>(maps, N, BH, Cpad, Nc, nA, nB, resident, G, labels,
                                                              done, changed, err, lost);
    }
    count_launches(1);
    SVGEAR_LAUNCH_CHECK();
    return SVGEAR_OK;
}

}  // namespace svgear
