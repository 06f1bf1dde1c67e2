// kmeans.cu -- k-means++ seeding, assignment, segment means and the
// permutation gather.
//
// Method: SVG2 (paper-graph summary, "Sparse VideoGen2 ...", section 3.4,
// "The clustering operation" and "Fast k-means with centroid cache"):
// independent k-means over the query and the key tokens of every head,
// k-means++ seeding for a cold start, centroid = mean of members; the
// permutation that makes clusters contiguous ("The permutation operation").
// The SVG-EAR task page (sotabase FrontierCS-2, agent step 1) adds that the
// k-means returns the sorted order and that a small kernel averages each
// cluster's values in one pass.
//
// B200 design: every pass over a token tensor moves 16-byte chunks with a
// group of lanes per token row (coalesced 128-bit loads); the assignment is a
// register-tiled fp32 contraction (tokens x centroids) with the argmin fused
// into its epilogue, so labels are the only output.
#include "common.cuh"
#include "launchers.h"

namespace svgear {

// ---------------------------------------------------------------------------
// k-means++: per pass j, (1) D^2 <- min(D^2, |x - seed_{j-1}|^2) with a
// deterministic fp64 scan per block of kKppTokens tokens, (2) one block per
// head locates the token where the running sum crosses u_j * sum(D^2).
// ---------------------------------------------------------------------------
constexpr int kKppThreads = 256;

// Inclusive fp64 prefix of 1024 fp32 values (4 per thread, token order) with
// a fixed reduction structure, so every call on the same values gives the
// same bits.  incl_tok receives the prefix at each of the thread's 4 tokens.
__device__ inline void kpp_block_scan(const float* d2s, double* warp_tot,
                                      double incl_tok[4]) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    double s[4], run = 0.0;
#pragma unroll
    for (int i = 0; i < 4; ++i) { run += (double)d2s[tid * 4 + i]; s[i] = run; }
    double x = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        double y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    double ex = __shfl_up_sync(0xffffffffu, x, 1);
    if (lane == 0) ex = 0.0;
    if (lane == 31) warp_tot[warp] = x;
    __syncthreads();
    double wbase = 0.0;
    for (int w = 0; w < warp; ++w) wbase += warp_tot[w];
    double base = wbase + ex;
#pragma unroll
    for (int i = 0; i < 4; ++i) incl_tok[i] = base + s[i];
}

template <typename T>
__global__ void kpp_first_kernel(const T* __restrict__ X, int N, int D, int C,
                                 uint64_t seed, uint64_t sbase, int32_t* chosen, float* centroids) {
    const int bh = blockIdx.x;
    double u = philox_uniform(seed, sbase + (uint64_t)bh, 0);
    long long t = (long long)floor(u * (double)N);
    if (t >= N) t = N - 1;
    if (threadIdx.x == 0) chosen[(size_t)bh * C] = (int32_t)t;
    const T* row = X + ((size_t)bh * N + t) * D;
    for (int k = threadIdx.x; k < D; k += blockDim.x)
        centroids[(size_t)bh * C * D + k] = Elem<T>::from(row[k]);
}

// Pick of seed j for head bh from the D^2 of this pass (run by the last block
// of the pass to finish): the block where the running sum of the block sums
// crosses u_j * sum, then the token inside it, with the same fp64 scan the
// blocks used, so the two levels agree bit for bit.  Also leaves in cc2 the
// squared distances from seed j to seeds 0..j-1 for the next pass's pruning.
template <typename T, int D>
__device__ void kpp_pick(const T* __restrict__ X, int N, int nblk, int bh, int32_t* chosen, int C,
                         int j, const float* D2, const double* blocksum, uint64_t seed,
                         uint64_t sbase,
                         float* centroids, float* cc2, float* d2s, double* warp_tot, float* cnew) {
    __shared__ int s_blk, s_pick, s_last;
    __shared__ double s_base, s_target;
    const int tid = threadIdx.x;
    const double* bs = blocksum + (size_t)bh * nblk;
    const float* d2 = D2 + (size_t)bh * N;
    int32_t* ch = chosen + (size_t)bh * C;
    // the block sums, fetched in parallel (the d2s buffer holds 512 doubles);
    // heads with more blocks than that read the rest from L2 in the loop below
    double* bsum = reinterpret_cast<double*>(d2s);
    constexpr int kCached = kKppTokens / 2;
    for (int b = tid; b < nblk && b < kCached; b += kKppThreads) bsum[b] = __ldcg(bs + b);
    __syncthreads();
    if (tid < 32) {
        // Lane l owns the block sums [l*per, l*per + per).  The running sum at
        // block b of lane l's chunk is E_l + (the chunk's sequential partial
        // sum through b), E_l the exclusive shuffle scan of the chunk totals:
        // a fixed structure, so the pick is the same on every run.
        const int lane = tid, per = (nblk + 31) / 32;
        const int b0 = min(lane * per, nblk), b1 = min(b0 + per, nblk);
        double c = 0.0;
        for (int b = b0; b < b1; ++b) c += b < kCached ? bsum[b] : __ldcg(bs + b);
        double x = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const double y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        double E = __shfl_up_sync(0xffffffffu, x, 1);
        if (lane == 0) E = 0.0;
        const double endv = E + c;
        const double total = __shfl_sync(0xffffffffu, endv, 31);
        int hit = -3;               // every D^2 is zero
        double base = 0.0, target = 0.0;
        if (total > 0.0) {
            target = philox_uniform(seed, sbase + (uint64_t)bh, (uint64_t)j) * total;
            const unsigned m = __ballot_sync(0xffffffffu, b1 > b0 && endv > target);
            hit = -2;               // rounding left no block above the target
            if (m) {
                const int src = __ffs(m) - 1;
                int h = b1 - 1;     // the chunk's end value is above the target
                double prev = E, part = 0.0;
                if (lane == src) {
                    for (int b = b0; b < b1; ++b) {
                        part += b < kCached ? bsum[b] : __ldcg(bs + b);
                        const double run = E + part;
                        if (run > target) { h = b; break; }
                        prev = run;
                    }
                }
                hit = __shfl_sync(0xffffffffu, h, src);
                base = __shfl_sync(0xffffffffu, prev, src);
            }
        }
        if (lane == 0) {
            s_pick = 0x7fffffff;
            s_last = -1;
            s_blk = hit;
            s_base = base;
            s_target = target;
        }
    }
    __syncthreads();
    const int blk = s_blk;
    if (blk >= 0) {
        for (int r = tid; r < kKppTokens; r += kKppThreads) {
            const int t = blk * kKppTokens + r;
            d2s[r] = (t < N) ? __ldcg(d2 + t) : 0.f;
        }
        __syncthreads();
        double incl[4];
        kpp_block_scan(d2s, warp_tot, incl);
        for (int i = 0; i < 4; ++i) {
            if (s_base + incl[i] > s_target) {
                atomicMin(&s_pick, blk * kKppTokens + tid * 4 + i);
                break;
            }
        }
        __syncthreads();
        if (s_pick == 0x7fffffff) {
            // the block-level and token-level sums rounded apart and no token
            // of the block reaches the target: take its last token with D^2 > 0
            for (int i = 0; i < 4; ++i)
                if (d2s[tid * 4 + i] > 0.f) atomicMax(&s_last, blk * kKppTokens + tid * 4 + i);
            __syncthreads();
            if (tid == 0 && s_last >= 0) s_pick = s_last;
            __syncthreads();
        }
    } else if (tid == 0) {
        int pick = 0;
        if (blk == -2) {            // rounding left no token above the target
            for (int t = N - 1; t >= 0; --t)
                if (__ldcg(d2 + t) > 0.f) { pick = t; break; }
        } else {                    // every D^2 is zero: lowest unchosen token
            for (int t = 0; t < N; ++t) {
                bool used = false;
                for (int q = 0; q < j; ++q) used |= (__ldcg(ch + q) == t);
                if (!used) { pick = t; break; }
            }
        }
        s_pick = pick;
    }
    __syncthreads();
    const int pick = s_pick < N ? s_pick : N - 1;
    if (tid == 0) ch[j] = pick;
    const T* row = X + ((size_t)bh * N + pick) * D;
    for (int k = tid; k < D; k += kKppThreads) {
        const float v = Elem<T>::from(row[k]);
        cnew[k] = v;
        centroids[((size_t)bh * C + j) * D + k] = v;
    }
    __syncthreads();
    // |c_j - c_a|^2 for a < j, one earlier seed per thread.  Seeds are rows
    // of X, so the distances read those rows in X's own type (half the bytes
    // of the fp32 centroid rows for bf16 inputs); this is the pass's latency
    // tail, bound by the loads one thread keeps in flight.
    constexpr int EPC = Elem<T>::kPerChunk;
    constexpr int NCH = D / EPC;
    const T* Xh = X + (size_t)bh * N * D;
    for (int a = tid; a < j; a += kKppThreads) {
        const T* ra = Xh + (size_t)__ldcg(ch + a) * D;
        float acc = 0.f;
#pragma unroll 8
        for (int k = 0; k < NCH; ++k) {
            float v[EPC];
            Elem<T>::unpack(Elem<T>::load_raw(ra + k * EPC), v);
#pragma unroll
            for (int e = 0; e < EPC; ++e) {
                const float df = v[e] - cnew[k * EPC + e];
                acc = fmaf(df, df, acc);
            }
        }
        cc2[(size_t)bh * C + a] = acc;
    }
}

// A token whose nearest seed a lies at squared distance cc2[a] >= kKppPrune *
// D^2 from the new seed s keeps its D^2: by the triangle inequality
// |x - c_s| >= |c_s - c_a| - |x - c_a| >= |x - c_a| once |c_s - c_a| >=
// 2 |x - c_a|.  The factor 4 (1 + 2^-7) leaves a margin far above the fp32
// rounding of either squared distance (a few units in 2^-24 per term summed),
// so a pruned token's recomputed fp32 distance would never have been below
// its D^2 and the pass stays bit-identical to the unpruned one.  A NaN fails
// the comparison and is recomputed.
constexpr float kKppPrune = 4.03125f;

// Shared memory of one k-means++ CTA.
template <int D>
struct KppSmem {
    float cen[D];                              // the seed this pass adds, fp32
    __align__(16) float d2s[kKppTokens];       // a block's D^2; also the pick's fp64 block sums
    int32_t todo[kKppTokens];                  // tokens of the block left by the screen
    double warp_tot[kKppThreads / 32];
    int ntodo;
};

// One 1024-token block of the pass adding seed s: D^2 <- min(D^2, |x - c_s|^2)
// and the block's fp64 scan total.  Tokens are first screened with the
// triangle bound (8 bytes read per token: D^2 and nearest-seed index); only
// the survivors' rows are loaded, by groups of lanes, four rows in flight.
template <typename T, int D>
__device__ void kpp_block_update(const T* __restrict__ X, int N, int nblk, int bh, int blk, int s,
                                 float* D2, int32_t* nearest, double* blocksum, KppSmem<D>& sm,
                                 const float* ccs) {
    constexpr int EPC = Elem<T>::kPerChunk;
    constexpr int L = D / EPC;                 // lanes per token row
    constexpr int RP = kKppThreads / L;        // rows per sweep of the block
    constexpr int U = 4;                       // rows in flight per lane group
    constexpr int TPT = kKppTokens / kKppThreads;   // tokens per thread
    const int tid = threadIdx.x, wl = tid & 31;
    const T* Xh = X + (size_t)bh * N * D;
    float* D2h = D2 + (size_t)bh * N;
    int32_t* nh = nearest + (size_t)bh * N;
    float dpre[TPT];
    int apre[TPT];
#pragma unroll
    for (int i = 0; i < TPT; ++i) {
        const int t = blk * kKppTokens + i * kKppThreads + tid;
        dpre[i] = 0.f;
        apre[i] = -1;
        if (t < N && s > 0) {
            dpre[i] = D2h[t];
            apre[i] = nh[t];
        }
    }
    if (tid == 0) sm.ntodo = 0;
    __syncthreads();
    // screen
#pragma unroll
    for (int i = 0; i < TPT; ++i) {
        const int r = i * kKppThreads + tid, t = blk * kKppTokens + r;
        float d = 0.f;
        bool need = false;
        if (t < N) {
            if (s == 0) {
                need = true;
            } else {
                d = dpre[i];
                const int a = apre[i];
                need = (unsigned)a >= (unsigned)s || !(ccs[a] >= kKppPrune * d);
            }
        }
        sm.d2s[r] = d;
        const unsigned m = __ballot_sync(0xffffffffu, need);
        int base = 0;
        if (wl == 0 && m) base = atomicAdd(&sm.ntodo, __popc(m));
        base = __shfl_sync(0xffffffffu, base, 0);
        if (need) sm.todo[base + __popc(m & ((1u << wl) - 1u))] = r;
    }
    __syncthreads();
    const int32_t* list = sm.todo;
    const int n = sm.ntodo;
    // recompute the survivors
    const int lane = tid % L, grp = tid / L;
    for (int b0 = 0; b0 < n; b0 += RP * U) {
        int rr[U];
        uint4 raw[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = b0 + grp + u * RP;
            rr[u] = i < n ? list[i] : -1;
            raw[u] = make_uint4(0u, 0u, 0u, 0u);
            if (rr[u] >= 0)
                raw[u] = Elem<T>::load_raw(Xh + (size_t)(blk * kKppTokens + rr[u]) * D + lane * EPC);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            float x[EPC];
            Elem<T>::unpack(raw[u], x);
            float part = 0.f;
#pragma unroll
            for (int e = 0; e < EPC; ++e) {
                const float df = x[e] - sm.cen[lane * EPC + e];
                part = fmaf(df, df, part);
            }
#pragma unroll
            for (int o = L / 2; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
            if (lane == 0 && rr[u] >= 0) {
                const int r = rr[u], t = blk * kKppTokens + r;
                const float old = sm.d2s[r];
                const float v = s == 0 ? part : fminf(part, old);
                if (s == 0 || __float_as_int(v) != __float_as_int(old)) {
                    sm.d2s[r] = v;
                    D2h[t] = v;
                    nh[t] = s;
                }
            }
        }
    }
    __syncthreads();
    double incl[4];
    kpp_block_scan(sm.d2s, sm.warp_tot, incl);
    if (tid == kKppThreads - 1) blocksum[(size_t)bh * nblk + blk] = incl[3];
    __syncthreads();   // d2s and warp_tot are reused by the next block
}

// Persistent seeding over a shared pool of work: every CTA serves every head.
// Head h's state is claim[h] (pass index p in the high 32 bits, blocks claimed
// in that pass in the low 32) and arrive[h] (blocks of pass p finished).  A
// CTA claims a 1024-token block of pass p (which adds seed p-1) from its own
// head c % BH first and from the other heads when that one has none left,
// processes it and arrives; the CTA that finishes the last block of the pass
// picks seed p (and the seed-to-seed distances of the next screen), resets
// arrive[h] and publishes pass p+1 by swapping claim[h] to (p+1) << 32.  No
// CTA waits for a particular head or CTA: while one head's pick runs, its
// CTAs work on the other heads' passes.  Every block's arithmetic is the same
// whichever CTA runs it, so the result does not depend on the schedule.  A
// CTA that finds no block anywhere for kKppWaitNs gives up with
// SVGEAR_ERR_TIMEOUT (err[1] = pass of its own head, err[2] = CTA).
constexpr uint64_t kKppWaitNs = 2000000000ull;

__device__ __forceinline__ uint64_t tc_global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

template <typename T, int D>
__global__ void __launch_bounds__(kKppThreads, 6)
kpp_pool_kernel(const T* __restrict__ X, int N, int nblk, int BH, int C, int32_t* chosen,
                float* D2, int32_t* nearest, float* cc2, double* blocksum,
                unsigned long long* claim, int32_t* arrive, int32_t* heads_done, uint64_t seed,
                uint64_t sbase, float* centroids, int* err) {
    __shared__ KppSmem<D> sm;
    extern __shared__ float ccs[];             // |c_s - c_a|^2, a < s (dynamic: C floats)
    __shared__ int s_bh, s_pass, s_blk, s_last;
    const int tid = threadIdx.x;
    const int home = blockIdx.x % BH;
    int cur_bh = -1, cur_pass = -1;            // seed row and screen distances in shared memory
    for (;;) {
        if (tid < 32) {
            // warp 0 looks for a block: lane l reads head home + l (+ 32 k), a
            // ballot picks the nearest head with unclaimed blocks, its lane claims
            const int lane = tid;
            int fbh = -1, fpass = 0, fblk = 0;
            const uint64_t t0 = tc_global_ns();
            for (;;) {
                int stop = 0;
                if (lane == 0) {
                    if (*(volatile int*)err != 0) stop = -2;
                    else if (*(volatile int*)heads_done >= BH) stop = -3;
                }
                stop = __shfl_sync(0xffffffffu, stop, 0);
                if (stop) { fbh = stop; break; }
                for (int k0 = 0; k0 < BH && fbh < 0; k0 += 32) {
                    const int k = k0 + lane;
                    int h = home + k;
                    if (h >= BH) h -= BH;
                    bool open = false;
                    if (k < BH) {
                        const unsigned long long w = *(volatile unsigned long long*)(claim + h);
                        open = (int)(w >> 32) < C && (uint32_t)w < (uint32_t)nblk;
                    }
                    unsigned m = __ballot_sync(0xffffffffu, open);
                    while (m && fbh < 0) {
                        const int src = __ffs(m) - 1;
                        m &= m - 1;
                        int got_bh = -1, got_pass = 0, got_blk = 0;
                        if (lane == src) {
                            const unsigned long long got = atomicAdd(claim + h, 1ull);
                            if ((int)(got >> 32) < C && (uint32_t)got < (uint32_t)nblk) {
                                got_bh = h;
                                got_pass = (int)(got >> 32);
                                got_blk = (int)(uint32_t)got;
                            }
                        }
                        got_bh = __shfl_sync(0xffffffffu, got_bh, src);
                        if (got_bh >= 0) {
                            fbh = got_bh;
                            fpass = __shfl_sync(0xffffffffu, got_pass, src);
                            fblk = __shfl_sync(0xffffffffu, got_blk, src);
                        }
                    }
                }
                if (fbh >= 0) break;
                // lane 0 alone reads the clock, so the warp leaves together
                const int expired = __shfl_sync(0xffffffffu,
                                                lane == 0 && tc_global_ns() - t0 > kKppWaitNs, 0);
                if (expired) {
                    if (lane == 0 && atomicCAS(err, 0, SVGEAR_ERR_TIMEOUT) == 0) {
                        err[1] = (int)(*(volatile unsigned long long*)(claim + home) >> 32);
                        err[2] = (int)blockIdx.x;
                    }
                    fbh = -2;
                    break;
                }
                __nanosleep(128);
            }
            __threadfence();   // acquire: the pick that published this pass is visible
            if (lane == 0) {
                s_bh = fbh;
                s_pass = fpass;
                s_blk = fblk;
            }
        }
        __syncthreads();
        const int bh = s_bh, pass = s_pass, blk = s_blk;
        if (bh < 0) return;
        const int s = pass - 1;
        if (bh != cur_bh || pass != cur_pass) {
            for (int k = tid; k < D; k += kKppThreads)
                sm.cen[k] = __ldcg(centroids + ((size_t)bh * C + s) * D + k);
            for (int a = tid; a < s; a += kKppThreads) ccs[a] = __ldcg(cc2 + (size_t)bh * C + a);
            cur_bh = bh;
            cur_pass = pass;
            // (the block update's first barrier orders these loads before their use)
        }
        kpp_block_update<T, D>(X, N, nblk, bh, blk, s, D2, nearest, blocksum, sm, ccs);
        // arrive; the block update's last barrier ordered its D^2, label and
        // block-sum stores before thread 0's fence
        if (tid == 0) {
            __threadfence();
            s_last = (atomicAdd(arrive + bh, 1) == nblk - 1);
        }
        __syncthreads();
        if (s_last) {
            __threadfence();
            kpp_pick<T, D>(X, N, nblk, bh, chosen, C, pass, D2, blocksum, seed, sbase, centroids, cc2,
                           sm.d2s, sm.warp_tot, sm.cen);
            __syncthreads();
            if (tid == 0) {
                arrive[bh] = 0;
                __threadfence();
                atomicExch(claim + bh, (unsigned long long)(pass + 1) << 32);   // release pass + 1
                if (pass + 1 >= C) atomicAdd(heads_done, 1);
            }
            cur_bh = -1;   // shared memory now holds the new seed, not the next screen's distances
        }
        __syncthreads();
    }
}

__global__ void kpp_init_kernel(unsigned long long* claim, int32_t* arrive, int32_t* heads_done,
                                int n) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) {
        claim[i] = 1ull << 32;   // pass 1: seed 0 comes from kpp_first_kernel, launched before
        arrive[i] = 0;
    }
    if (i == 0) *heads_done = 0;
}

template <typename T, int D>
static int kmeanspp_impl(const T* X, svgear_dims dims, int C, uint64_t seed, uint64_t sbase,
                         float* cent,
                         int32_t* chosen, float* D2, int32_t* nearest, float* cc2,
                         double* blocksum, int32_t* counter, int32_t* gen, int* err,
                         cudaStream_t st) {
    const int BH = dims.B * dims.H, N = dims.N;
    const int nblk = ceil_div(N, kKppTokens);
    // the counter array (2 BH words) holds the heads' claim words, gen (BH + 1
    // words) the arrival counts and the finished-head count
    unsigned long long* claim = reinterpret_cast<unsigned long long*>(counter);
    int32_t* arrive = gen;
    int32_t* heads_done = gen + BH;
    kpp_init_kernel<<<ceil_div(BH, 128), 128, 0, st>>>(claim, arrive, heads_done, BH);
    count_launches(1);
    kpp_first_kernel<T><<<BH, 128, 0, st>>>(X, N, D, C, seed, sbase, chosen, cent);
    count_launches(1);
    SVGEAR_LAUNCH_CHECK();
    if (C < 2) return SVGEAR_OK;
    // every CTA resident (cooperative launch), as many as fit, at most one per
    // block of a pass over all heads
    int dev = 0, sms = 0, per_sm = 0;
    const size_t ccs_bytes = sizeof(float) * (size_t)C;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kpp_pool_kernel<T, D>,
                                                      kKppThreads, ccs_bytes) != cudaSuccess ||
        per_sm < 1)
        return SVGEAR_ERR_CUDA;
    long long grid = (long long)per_sm * sms;
    if (grid > (long long)BH * nblk) grid = (long long)BH * nblk;
    int n_ = N, nblk_ = nblk, BH_ = BH, C_ = C;
    uint64_t seed_ = seed, sbase_ = sbase;
    const T* X_ = X;
    void* args[] = {&X_, &n_, &nblk_, &BH_, &C_, &chosen, &D2, &nearest, &cc2, &blocksum,
                    &claim, &arrive, &heads_done, &seed_, &sbase_, &cent, &err};
    if (cudaLaunchCooperativeKernel((const void*)kpp_pool_kernel<T, D>, dim3((unsigned)grid),
                                    dim3(kKppThreads), args, ccs_bytes, st) != cudaSuccess)
        return SVGEAR_ERR_CUDA;
    count_launches(1);
    return SVGEAR_OK;
}

// ---------------------------------------------------------------------------
// Assignment: a 128-token x 128-centroid register-tiled fp32 contraction per
// step (256 threads, 8x8 per thread), distance |c|^2 - 2 x.c, argmin fused.
// The centroids are first re-laid k-major ([d][Cpad], Cpad a multiple of 128,
// padding norm = +inf), so each 32-deep chunk of a centroid tile is a plain
// 16-byte cp.async copy into shared memory, double-buffered behind the FMAs.
// ---------------------------------------------------------------------------
constexpr int kAsTM = 128, kAsTN = 128, kAsKC = 32, kAsThreads = 256;

__device__ __forceinline__ void cpa16(float* dst_smem, const float* src) {
    const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst_smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
}

// cT[bh][k][c] = cent[bh][c][k] (0 for padding), cn[bh][c] = |c|^2 (+inf for padding).
template <int D>
__global__ void centroid_kmajor_kernel(const float* __restrict__ cent, int C, int Cpad,
                                       float* __restrict__ cT, float* __restrict__ cn,
                                       const int32_t* __restrict__ done) {
    const int bh = blockIdx.y;
    if (done && done[bh]) return;
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= Cpad) return;
    const float* src = cent + ((size_t)bh * C + c) * D;
    float* dst = cT + (size_t)bh * D * Cpad + c;
    float s = 0.f;
    if (c < C) {
        for (int k = 0; k < D; ++k) {
            const float v = src[k];
            s = fmaf(v, v, s);
            dst[(size_t)k * Cpad] = v;
        }
        cn[(size_t)bh * Cpad + c] = s;
    } else {
        for (int k = 0; k < D; ++k) dst[(size_t)k * Cpad] = 0.f;
        cn[(size_t)bh * Cpad + c] = __int_as_float(0x7f800000);
    }
}

template <typename T, int D>
__global__ void __launch_bounds__(kAsThreads, 2)
assign_kernel(const T* __restrict__ X, int N, const float* __restrict__ cT,
              const float* __restrict__ cnorm, int C, int Cpad, int32_t* __restrict__ labels,
              const int32_t* __restrict__ done, int32_t* __restrict__ changed) {
    constexpr int EPC = Elem<T>::kPerChunk;
    constexpr int CPR = D / EPC;               // 16-byte chunks per token row
    extern __shared__ __align__(16) float smem[];
    float* Xs = smem;                          // [D][kAsTM] (transposed tile)
    float* Cs = Xs + D * kAsTM;                // [2][kAsKC][kAsTN]
    const int bh = blockIdx.y, t0 = blockIdx.x * kAsTM, tid = threadIdx.x;
    if (done && done[bh]) return;   // this head reached its fixed point
    const T* Xh = X + (size_t)bh * N * D;
    const float* cTh = cT + (size_t)bh * D * Cpad;
    const float* cnh = cnorm + (size_t)bh * Cpad;
    const int nchunks = (Cpad / kAsTN) * (D / kAsKC);

    // chunk n: centroid tile n / (D/kAsKC), depth slice n % (D/kAsKC)
    auto load_chunk = [&](int n, int buf) {
        const int c0 = (n / (D / kAsKC)) * kAsTN, k0 = (n % (D / kAsKC)) * kAsKC;
        float* dst = Cs + buf * kAsKC * kAsTN;
#pragma unroll
        for (int q = tid; q < kAsKC * kAsTN / 4; q += kAsThreads) {
            const int kk = q / (kAsTN / 4), cc = (q % (kAsTN / 4)) * 4;
            cpa16(dst + kk * kAsTN + cc, cTh + (size_t)(k0 + kk) * Cpad + c0 + cc);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    load_chunk(0, 0);

    // token tile, transposed; consecutive lanes take consecutive tokens so the
    // transposed shared-memory stores are conflict-free
    for (int q = tid; q < kAsTM * CPR; q += kAsThreads) {
        const int row = q % kAsTM, col = (q / kAsTM) * EPC;
        float v[EPC];
        if (t0 + row < N) Elem<T>::load(Xh + (size_t)(t0 + row) * D + col, v);
        else
#pragma unroll
            for (int e = 0; e < EPC; ++e) v[e] = 0.f;
#pragma unroll
        for (int e = 0; e < EPC; ++e) Xs[(col + e) * kAsTM + row] = v[e];
    }

    const int tx = tid & 15, ty = tid >> 4;
    float bestd[8];
    int besti[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) { bestd[i] = __int_as_float(0x7f800000); besti[i] = 0; }
    float acc[8][8];

    for (int n = 0; n < nchunks; ++n) {
        const int kslice = n % (D / kAsKC);
        if (n + 1 < nchunks) {
            load_chunk(n + 1, (n + 1) & 1);
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncthreads();
        if (kslice == 0) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) acc[i][jj] = 0.f;
        }
        const float* cbuf = Cs + (n & 1) * kAsKC * kAsTN;
        const int k0 = kslice * kAsKC;
#pragma unroll 4
        for (int k = 0; k < kAsKC; ++k) {
            const float* xr = Xs + (k0 + k) * kAsTM;
            const float* cr = cbuf + k * kAsTN;
            const float4 a0 = *reinterpret_cast<const float4*>(xr + ty * 4);
            const float4 a1 = *reinterpret_cast<const float4*>(xr + 64 + ty * 4);
            const float4 b0 = *reinterpret_cast<const float4*>(cr + tx * 4);
            const float4 b1 = *reinterpret_cast<const float4*>(cr + 64 + tx * 4);
            const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) acc[i][jj] = fmaf(a[i], b[jj], acc[i][jj]);
        }
        if (kslice == D / kAsKC - 1) {
            // candidates of this thread come in increasing centroid order
            const int c0 = (n / (D / kAsKC)) * kAsTN;
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                const int cj = (jj < 4) ? tx * 4 + jj : 64 + tx * 4 + (jj - 4);
                const float cnv = __ldg(cnh + c0 + cj);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float dist = fmaf(-2.f, acc[i][jj], cnv);
                    if (dist < bestd[i]) { bestd[i] = dist; besti[i] = c0 + cj; }
                }
            }
        }
        __syncthreads();   // buffer n&1 is refilled by the next iteration's load
    }
    // lexicographic (distance, index) minimum over the 16 threads of a row group
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float dd = bestd[i];
        int ix = besti[i];
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) {
            const float od = __shfl_xor_sync(0xffffffffu, dd, o);
            const int oi = __shfl_xor_sync(0xffffffffu, ix, o);
            if (od < dd || (od == dd && oi < ix)) { dd = od; ix = oi; }
        }
        if (tx == 0) {
            const int row = (i < 4) ? ty * 4 + i : 64 + ty * 4 + (i - 4);
            if (t0 + row < N) {
                int32_t* lp = labels + (size_t)bh * N + t0 + row;
                if (changed && *lp != ix) changed[bh] = 1;
                *lp = ix;
            }
        }
    }
}

template <typename T, int D>
static int assign_impl(const T* X, svgear_dims dims, const float* cent, int C,
                       int32_t* labels, const int32_t* done, int32_t* changed, float* cT,
                       float* cnorm, cudaStream_t st) {
    const int Cpad = ceil_div(C, kAsTN) * kAsTN;
    const int BH = dims.B * dims.H;
    centroid_kmajor_kernel<D><<<dim3(ceil_div(Cpad, 128), BH), 128, 0, st>>>(cent, C, Cpad, cT, cnorm,
                                                                             done);
    count_launches(1);
    const size_t smem = sizeof(float) * (D * kAsTM + 2 * kAsKC * kAsTN);
    // per-device function attribute; cheap enough to set on every call
    if (cudaFuncSetAttribute(assign_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
        return SVGEAR_ERR_CUDA;
    assign_kernel<T, D><<<dim3(ceil_div(dims.N, kAsTM), BH), kAsThreads, smem, st>>>(
        X, dims.N, cT, cnorm, C, Cpad, labels, done, changed);
    count_launches(1);
    SVGEAR_LAUNCH_CHECK();
    return SVGEAR_OK;
}

size_t assign_scratch_bytes(int BH, int C, int D, int dtype) {
    if (dtype == SVGEAR_BF16) return assign_sm100_scratch_bytes(BH, C, D);
    const size_t Cpad = (size_t)ceil_div(C, kAsTN) * kAsTN;
    return (size_t)BH * Cpad * (D + 1) * sizeof(float);
}

// ---------------------------------------------------------------------------
// Segment mean (the k-means update and the per-cluster value means).
//
// Work is split by position, not by segment, so every CTA moves the same
// bytes whatever the cluster sizes: CTA (j, bh) takes the permuted positions
// [jP, (j+1)P) of head bh.  The segments crossing that range are summed one
// piece at a time (a piece = a segment's positions inside the chunk): lane
// group g of the CTA adds the rows r0+g, r0+g+R, ... of the piece in order
// (fp32), and the R group sums are added in group order.  A segment inside
// one chunk is finished there; a longer one leaves its first piece as the
// chunk's "trail" partial and the others as "lead" partials of the following
// chunks, and segment_join_kernel adds trail(j0) + lead(j0+1) + ... +
// lead(j1) in that order.  The summation order is a function of the
// positions alone, so results are identical from run to run and for any
// grid.  An empty segment writes zeros (empty_zero) or keeps its row.
// Gather mode reads row perm[p] at position p; the chunk's perm entries are
// staged in shared memory first, so no row load waits on an index load.
// ---------------------------------------------------------------------------
constexpr int kSmThreads = 256;
constexpr int kSmChunk = 512;   // positions per CTA (128 KB of bf16 d = 128 rows)
constexpr int kSmUnroll = 8;    // rows in flight per lane group

size_t segmean_scratch_bytes(int BH, int N, int D) {
    const size_t nch = (size_t)ceil_div(N, kSmChunk);
    return (size_t)BH * nch * (2 * (size_t)D * sizeof(float) + sizeof(int32_t)) + 3 * 256;
}

// Segment containing position p (offsets non-decreasing, offsets[0] = 0,
// offsets[C] = N, p < N): the last c with offsets[c] <= p, skipping empties
// (their offsets[c] == offsets[c + 1] <= p).
__device__ __forceinline__ int segment_of(const int32_t* off, int C, int p) {
    int lo = 0, hi = C - 1;   // invariant: off[lo] <= p < off[hi + 1]
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (off[mid] <= p) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

template <typename T, int D, bool GATHER>
__global__ void __launch_bounds__(kSmThreads)
segment_piece_kernel(const T* __restrict__ X, const int32_t* __restrict__ perm,
                     const int32_t* __restrict__ offsets, int N, int C, float* __restrict__ out,
                     bool empty_zero, const int32_t* __restrict__ done, float* __restrict__ lead,
                     float* __restrict__ trail, int32_t* __restrict__ trail_seg) {
    constexpr int EPC = Elem<T>::kPerChunk;
    constexpr int L = D / EPC;          // lanes per row
    constexpr int R = kSmThreads / L;   // lane groups
    constexpr int U = kSmUnroll;
    __shared__ float part[R][D];
    __shared__ int32_t rows_s[GATHER ? kSmChunk : 1];
    const int j = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    const int nch = gridDim.x;
    if (done && done[bh]) return;
    const int32_t* off = offsets + (size_t)bh * (C + 1);
    const int c0 = j * kSmChunk, c1 = min(c0 + kSmChunk, N);
    const T* Xh = X + (size_t)bh * N * D;
    float* lead_j = lead + ((size_t)bh * nch + j) * D;
    float* trail_j = trail + ((size_t)bh * nch + j) * D;
    if (GATHER) {
        for (int p = c0 + tid; p < c1; p += kSmThreads) rows_s[p - c0] = perm[(size_t)bh * N + p];
    }
    int seg = segment_of(off, C, c0);
    const bool last_chunk = j == nch - 1;
    // empty segments: those c with off[c] == off[c+1] in [c0, c1) (or == N on
    // the last chunk) belong to this chunk
    if (empty_zero) {
        int e_lo = 0, hi = C;   // the first c whose offset is >= c0
        while (e_lo < hi) {
            const int mid = (e_lo + hi) >> 1;
            if (off[mid] < c0) e_lo = mid + 1;
            else hi = mid;
        }
        for (int c = e_lo; c < C; ++c) {
            const int a = off[c];
            if (a >= c1 && !(last_chunk && a == N)) break;
            if (off[c + 1] == a)
                for (int k = tid; k < D; k += kSmThreads) out[((size_t)bh * C + c) * D + k] = 0.f;
        }
    }
    if (tid == 0) trail_seg[(size_t)bh * nch + j] = -1;
    __syncthreads();
    const int lane = tid % L, grp = tid / L;
    for (int p0 = c0; p0 < c1;) {
        const int a = off[seg], b = off[seg + 1];
        if (b <= p0 || a > p0) break;          // malformed offsets: stop rather than spin
        const int r0 = p0, r1 = min(b, c1);   // this piece
        float acc[EPC];
#pragma unroll
        for (int e = 0; e < EPC; ++e) acc[e] = 0.f;
        // U rows in flight per lane group, all loads before the first add;
        // a slot past the piece reloads the piece's first row and is not
        // added (nor is a gathered row outside the head: malformed perm)
        for (int p = r0 + grp; p < r1; p += U * R) {
            int row[U];
            uint4 v[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int q = p + u * R;
                const int at = q < r1 ? q : r0;
                const int rr = GATHER ? rows_s[at - c0] : at;
                row[u] = q < r1 ? rr : -1;
                const int rc = GATHER ? min(max(rr, 0), N - 1) : rr;
                v[u] = Elem<T>::load_raw(Xh + (size_t)rc * D + lane * EPC);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if ((unsigned)row[u] >= (unsigned)N) continue;
                float f[EPC];
                Elem<T>::unpack(v[u], f);
#pragma unroll
                for (int e = 0; e < EPC; ++e) acc[e] += f[e];
            }
        }
#pragma unroll
        for (int e = 0; e < EPC; ++e) part[grp][lane * EPC + e] = acc[e];
        __syncthreads();
        for (int k = tid; k < D; k += kSmThreads) {
            float s = 0.f;
#pragma unroll
            for (int g = 0; g < R; ++g) s += part[g][k];
            if (a < c0) lead_j[k] = s;                 // started in an earlier chunk
            else if (b > c1) trail_j[k] = s;           // continues in later chunks
            else out[((size_t)bh * C + seg) * D + k] = s / (float)(b - a);
        }
        if (tid == 0 && a >= c0 && b > c1) trail_seg[(size_t)bh * nch + j] = seg;
        __syncthreads();
        p0 = r1;
        if (p0 < c1) {   // next non-empty segment
            if (++seg >= C) break;
            while (seg < C - 1 && off[seg + 1] <= p0) ++seg;
        }
    }
}

// Segments longer than one chunk: trail(j0) + lead(j0+1) + ... + lead(j1).
template <int D>
__global__ void segment_join_kernel(const int32_t* __restrict__ offsets, int N, int C,
                                    float* __restrict__ out, const int32_t* __restrict__ done,
                                    const float* __restrict__ lead,
                                    const float* __restrict__ trail,
                                    const int32_t* __restrict__ trail_seg) {
    const int j = blockIdx.x, bh = blockIdx.y, k = threadIdx.x;
    const int nch = gridDim.x;
    if (done && done[bh]) return;
    const int c = trail_seg[(size_t)bh * nch + j];
    if (c < 0 || c >= C) return;
    const int32_t* off = offsets + (size_t)bh * (C + 1);
    const int a = off[c], b = off[c + 1];
    const int j1 = min((b - 1) / kSmChunk, nch - 1);
    float s = trail[((size_t)bh * nch + j) * D + k];
    for (int jj = j + 1; jj <= j1; ++jj) s += lead[((size_t)bh * nch + jj) * D + k];
    out[((size_t)bh * C + c) * D + k] = s / (float)(b - a);
}

// ---------------------------------------------------------------------------
// Per-coordinate variance of every segment (SVG-EAR blog, variance paragraph:
// one variance per key coordinate): out[c][k] = (1/n) sum_t (x_tk - mean_ck)^2
// over the contiguous rows of segment c, the mean taken first (two passes,
// fp32 partial sums combined in a fixed order); an empty segment gets 0.
// ---------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(kSmThreads)
segment_var_kernel(const T* __restrict__ X, const int32_t* __restrict__ offsets, int N, int C,
                   float* __restrict__ out) {
    constexpr int EPC = Elem<T>::kPerChunk;
    constexpr int L = D / EPC;
    constexpr int R = kSmThreads / L;
    __shared__ float part[R][D];
    __shared__ float mean[D];
    const int c = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    const int32_t* off = offsets + (size_t)bh * (C + 1);
    const int a = off[c], b = off[c + 1];
    float* o = out + ((size_t)bh * C + c) * D;
    if (b <= a || a < 0 || b > N) {
        for (int k = tid; k < D; k += kSmThreads) o[k] = 0.f;
        return;
    }
    const T* Xh = X + (size_t)bh * N * D;
    const int lane = tid % L, grp = tid / L;
    const float n = (float)(b - a);
    for (int pass = 0; pass < 2; ++pass) {
        float acc[EPC];
#pragma unroll
        for (int e = 0; e < EPC; ++e) acc[e] = 0.f;
        for (int p = a + grp; p < b; p += R) {
            float v[EPC];
            Elem<T>::load(Xh + (size_t)p * D + lane * EPC, v);
#pragma unroll
            for (int e = 0; e < EPC; ++e) {
                if (pass == 0) {
                    acc[e] += v[e];
                } else {
                    const float dv = v[e] - mean[lane * EPC + e];
                    acc[e] = fmaf(dv, dv, acc[e]);
                }
            }
        }
#pragma unroll
        for (int e = 0; e < EPC; ++e) part[grp][lane * EPC + e] = acc[e];
        __syncthreads();
        for (int k = tid; k < D; k += kSmThreads) {
            float s = 0.f;
#pragma unroll
            for (int g = 0; g < R; ++g) s += part[g][k];
            if (pass == 0) mean[k] = s / n;
            else o[k] = s / n;
        }
        __syncthreads();
    }
}

template <typename T, int D>
static int segvar_disp(const void* X, const int32_t* offsets, int C, svgear_dims dims, float* out,
                       cudaStream_t st) {
    segment_var_kernel<T, D><<<dim3(C, dims.B * dims.H), kSmThreads, 0, st>>>(
        static_cast<const T*>(X), offsets, dims.N, C, out);
    count_launches(1);
    SVGEAR_LAUNCH_CHECK();
    return SVGEAR_OK;
}

// ---------------------------------------------------------------------------
// Permutation gather: Xp[p] = X[perm[p]], one 16-byte chunk per thread.
// ---------------------------------------------------------------------------
template <typename T, int D>
__global__ void permute_kernel(const T* __restrict__ X, const int32_t* __restrict__ perm,
                               int N, T* __restrict__ Xp) {
    constexpr int EPC = Elem<T>::kPerChunk;
    constexpr int L = D / EPC;
    const int bh = blockIdx.y;
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long p = idx / L;
    const int lane = (int)(idx % L);
    if (p >= N) return;
    const int row = perm[(size_t)bh * N + p];
    if ((unsigned)row >= (unsigned)N) return;
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(X + ((size_t)bh * N + row) * D + lane * EPC));
    *reinterpret_cast<uint4*>(Xp + ((size_t)bh * N + p) * D + lane * EPC) = v;
}

// ---------------------------------------------------------------------------
// Dispatch on (dtype, d).
// ---------------------------------------------------------------------------
#define SVGEAR_DISPATCH(dims, FN, ...)                                              \
    do {                                                                             \
        if ((dims).dtype == SVGEAR_BF16) {                                           \
            if ((dims).d == 128) return FN<__nv_bfloat16, 128>(__VA_ARGS__);          \
            if ((dims).d == 64) return FN<__nv_bfloat16, 64>(__VA_ARGS__);            \
        } else if ((dims).dtype == SVGEAR_F32) {                                     \
            if ((dims).d == 128) return FN<float, 128>(__VA_ARGS__);                  \
            if ((dims).d == 64) return FN<float, 64>(__VA_ARGS__);                    \
        }                                                                            \
        return SVGEAR_ERR_UNSUPPORTED;                                               \
    } while (0)

template <typename T, int D>
static int kmeanspp_disp(const void* X, svgear_dims dims, int C, uint64_t seed, uint64_t sbase,
                         float* cent,
                         int32_t* chosen, float* D2, int32_t* nearest, float* cc2, double* bs,
                         int32_t* counter, int32_t* gen, int* err, cudaStream_t st) {
    return kmeanspp_impl<T, D>(static_cast<const T*>(X), dims, C, seed, sbase, cent, chosen, D2,
                               nearest,
                               cc2, bs, counter, gen, err, st);
}
int launch_kmeanspp(const void* X, svgear_dims dims, int C, uint64_t seed, uint64_t sbase,
                    float* cent,
                    int32_t* chosen, float* D2, int32_t* nearest, float* cc2, double* bs,
                    int32_t* counter, int32_t* gen, int* err, cudaStream_t st) {
    SVGEAR_DISPATCH(dims, kmeanspp_disp, X, dims, C, seed, sbase, cent, chosen, D2, nearest, cc2, bs,
                    counter, gen, err, st);
}

template <typename T, int D>
static int assign_disp(const void* X, svgear_dims dims, const float* cent, int C,
                       int32_t* labels, const int32_t* done, int32_t* changed, void* scratch,
                       int* err, cudaStream_t st) {
    if (dims.dtype == SVGEAR_BF16)
        return launch_assign_sm100(X, dims, cent, C, labels, scratch, err, st, done, changed);
    const size_t Cpad = (size_t)ceil_div(C, kAsTN) * kAsTN;
    float* cT = static_cast<float*>(scratch);
    float* cn = cT + (size_t)dims.B * dims.H * Cpad * D;
    return assign_impl<T, D>(static_cast<const T*>(X), dims, cent, C, labels, done, changed, cT,
                             cn, st);
}
int launch_assign(const void* X, svgear_dims dims, const float* cent, int C, int32_t* labels,
                  void* scratch, int* err, cudaStream_t st, const int32_t* done,
                  int32_t* changed) {
    SVGEAR_DISPATCH(dims, assign_disp, X, dims, cent, C, labels, done, changed, scratch, err, st);
}

// A head whose assignment changed no label has reached the fixed point of
// Lloyd's iteration: its (deterministic) update would reproduce the current
// centroids, so every later round is a no-op for it.
__global__ void kmeans_fixed_point_kernel(int32_t* __restrict__ changed, int32_t* __restrict__ done,
                                          int BH) {
    const int bh = blockIdx.x * blockDim.x + threadIdx.x;
    if (bh >= BH) return;
    if (!changed[bh]) done[bh] = 1;
    changed[bh] = 0;
}

int launch_fixed_point(int32_t* changed, int32_t* done, int BH, cudaStream_t st) {
    kmeans_fixed_point_kernel<<<ceil_div(BH, 128), 128, 0, st>>>(changed, done, BH);
    count_launches(1);
    SVGEAR_LAUNCH_CHECK();
    return SVGEAR_OK;
}

template <typename T, int D>
static int segmean_disp(const void* X, const int32_t* perm, const int32_t* offsets, int C,
                        svgear_dims dims, float* out, bool empty_zero, const int32_t* done,
                        void* scratch, cudaStream_t st) {
    const int BH = dims.B * dims.H;
    const int nch = ceil_div(dims.N, kSmChunk);
    const size_t parts = (size_t)BH * nch * D;
    float* lead = static_cast<float*>(scratch);
    float* trail = lead + parts;
    int32_t* tseg = reinterpret_cast<int32_t*>(trail + parts);
    if (perm)
        segment_piece_kernel<T, D, true><<<dim3(nch, BH), kSmThreads, 0, st>>>(
            static_cast<const T*>(X), perm, offsets, dims.N, C, out, empty_zero, done, lead,
            trail, tseg);
    else
        segment_piece_kernel<T, D, false><<<dim3(nch, BH), kSmThreads, 0, st>>>(
            static_cast<const T*>(X), nullptr, offsets, dims.N, C, out, empty_zero, done, lead,
            trail, tseg);
    segment_join_kernel<D><<<dim3(nch, BH), D, 0, st>>>(offsets, dims.N, C, out, done, lead, trail,
                                                       tseg);
    count_launches(2);
    SVGEAR_LAUNCH_CHECK();
    return SVGEAR_OK;
}
int launch_segment_mean(const void* X, const int32_t* perm, const int32_t* offsets, int C,
                        svgear_dims dims, float* out, bool empty_zero, void* scratch,
                        cudaStream_t st, const int32_t* done) {
    SVGEAR_DISPATCH(dims, segmean_disp, X, perm, offsets, C, dims, out, empty_zero, done, scratch,
                    st);
}

template <typename T, int D>
static int permute_disp(const void* X, const int32_t* perm, svgear_dims dims, void* Xp,
                        cudaStream_t st) {
    constexpr int L = D / Elem<T>::kPerChunk;
    const int BH = dims.B * dims.H;
    const long long chunks = (long long)dims.N * L;
    permute_kernel<T, D><<<dim3(ceil_div(chunks, 256), BH), 256, 0, st>>>(
        static_cast<const T*>(X), perm, dims.N, static_cast<T*>(Xp));
    count_launches(1);
    SVGEAR_LAUNCH_CHECK();
    return SVGEAR_OK;
}
int launch_permute(const void* X, const int32_t* perm, svgear_dims dims, void* Xp,
                   cudaStream_t st) {
    SVGEAR_DISPATCH(dims, permute_disp, X, perm, dims, Xp, st);
}

int launch_segment_var(const void* X, const int32_t* offsets, int C, svgear_dims dims,
                       float* out, cudaStream_t st) {
    SVGEAR_DISPATCH(dims, segvar_disp, X, offsets, C, dims, out, st);
}

}  // namespace svgear
