// sort.cu -- stable counting sort of cluster labels: the permutation that
// makes every cluster contiguous and the segment offsets.
//
// Method: SVG2 (paper-graph summary, section 3.4, "The permutation operation
// and its mathematical validity": tokens of cluster 1 first, then cluster 2,
// ...), and the SVG-EAR task page (agent step 1: the k-means also returns the
// sorted order).  Ties keep the original token order, so the result is
// unique and deterministic.
//
// Three passes per (batch, head): block histograms (shared-memory integer
// atomics), a column scan over blocks plus the segment offsets, and a
// one-warp-per-block scatter that ranks equal labels with __match_any_sync
// in token order.  Labels outside 0..C-1 are ignored (no write).
#include "common.cuh"
#include "launchers.h"

namespace svgear {

__global__ void sort_hist_kernel(const int32_t* __restrict__ labels, int N, int C, int nblk,
                                 int32_t* __restrict__ hist, const int32_t* __restrict__ done) {
    extern __shared__ int32_t h[];
    const int blk = blockIdx.x, bh = blockIdx.y;
    if (done && done[bh]) return;
    for (int c = threadIdx.x; c < C; c += blockDim.x) h[c] = 0;
    __syncthreads();
    const int32_t* lab = labels + (size_t)bh * N;
    for (int r = threadIdx.x; r < kSortTokens; r += blockDim.x) {
        const int t = blk * kSortTokens + r;
        if (t < N) {
            const int c = lab[t];
            if ((unsigned)c < (unsigned)C) atomicAdd(&h[c], 1);
        }
    }
    __syncthreads();
    int32_t* out = hist + ((size_t)bh * nblk + blk) * C;
    for (int c = threadIdx.x; c < C; c += blockDim.x) out[c] = h[c];
}

// hist[blk][c] <- number of tokens labelled c in blocks before blk (the
// start of block blk's run inside segment c); offsets <- the segment starts.
// One CTA per (batch, head).  A thread owns whole columns c; it loads a
// column 16 blocks at a time before storing any of them, so the loads of a
// column are in flight together.  The segment starts are an exclusive scan
// of the column totals: contiguous chunks per thread, then a shuffle scan of
// the chunk sums.
constexpr int kScanBatch = 16;
__global__ void sort_scan_kernel(int N, int C, int nblk, int32_t* __restrict__ hist,
                                 int32_t* __restrict__ offsets, const int32_t* __restrict__ done) {
    extern __shared__ int32_t tot[];   // [C] then [blockDim / 32] warp sums
    int32_t* wsum = tot + C;
    const int bh = blockIdx.x, tid = threadIdx.x, nt = blockDim.x;
    const int lane = tid & 31, warp = tid >> 5;
    if (done && done[bh]) return;
    int32_t* hh = hist + (size_t)bh * nblk * C;
    for (int c = tid; c < C; c += nt) {
        int32_t run = 0;
        for (int b0 = 0; b0 < nblk; b0 += kScanBatch) {
            int32_t v[kScanBatch];
#pragma unroll
            for (int u = 0; u < kScanBatch; ++u)
                v[u] = (b0 + u < nblk) ? hh[(size_t)(b0 + u) * C + c] : 0;
#pragma unroll
            for (int u = 0; u < kScanBatch; ++u) {
                if (b0 + u < nblk) hh[(size_t)(b0 + u) * C + c] = run;
                run += v[u];
            }
        }
        tot[c] = run;
    }
    __syncthreads();
    const int per = (C + nt - 1) / nt;
    const int c0 = min(C, tid * per), c1 = min(C, c0 + per);
    int32_t s = 0;
    for (int c = c0; c < c1; ++c) s += tot[c];
    int32_t x = s;   // inclusive scan of the chunk sums within the warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) wsum[warp] = x;
    __syncthreads();
    int32_t run = x - s;
    for (int w = 0; w < warp; ++w) run += wsum[w];
    int32_t* off = offsets + (size_t)bh * (C + 1);
    for (int c = c0; c < c1; ++c) { off[c] = run; run += tot[c]; }
    if (tid == nt - 1) off[C] = run;   // equals the number of in-range labels
}

__global__ void __launch_bounds__(32)
sort_scatter_kernel(const int32_t* __restrict__ labels, int N, int C, int nblk,
                    const int32_t* __restrict__ hist, const int32_t* __restrict__ offsets,
                    int32_t* __restrict__ perm, const int32_t* __restrict__ done) {
    extern __shared__ int32_t cur[];
    const int blk = blockIdx.x, bh = blockIdx.y, lane = threadIdx.x;
    if (done && done[bh]) return;
    const int32_t* hb = hist + ((size_t)bh * nblk + blk) * C;
    const int32_t* off = offsets + (size_t)bh * (C + 1);
    for (int c = lane; c < C; c += 32) cur[c] = off[c] + hb[c];
    __syncwarp();
    const int32_t* lab = labels + (size_t)bh * N;
    int32_t* pm = perm + (size_t)bh * N;
    const unsigned lt = (1u << lane) - 1u;
    for (int step = 0; step < kSortTokens / 32; ++step) {
        const int t = blk * kSortTokens + step * 32 + lane;
        int c = (t < N) ? lab[t] : -1;
        if ((unsigned)c >= (unsigned)C) c = -1;
        const unsigned same = __match_any_sync(0xffffffffu, c);
        int pos = 0;
        if (c >= 0) pos = cur[c] + __popc(same & lt);
        __syncwarp();
        if (c >= 0 && (same & lt) == 0) cur[c] += __popc(same);
        __syncwarp();
        if (c >= 0) pm[pos] = t;
    }
}

int launch_label_sort(const int32_t* labels, int BH, int N, int C, int32_t* perm,
                      int32_t* offsets, int32_t* hist, cudaStream_t st, const int32_t* done) {
    const int nblk = ceil_div(N, kSortTokens);
    const size_t sh = sizeof(int32_t) * C;
    sort_hist_kernel<<<dim3(nblk, BH), 256, sh, st>>>(labels, N, C, nblk, hist, done);
    count_launches(1);
    const int nt = 512;
    sort_scan_kernel<<<BH, nt, sizeof(int32_t) * (C + nt / 32), st>>>(N, C, nblk, hist, offsets,
                                                                      done);
    count_launches(1);
    sort_scatter_kernel<<<dim3(nblk, BH), 32, sh, st>>>(labels, N, C, nblk, hist, offsets, perm,
                                                        done);
    count_launches(1);
    SVGEAR_LAUNCH_CHECK();
    return SVGEAR_OK;
}

}  // namespace svgear
