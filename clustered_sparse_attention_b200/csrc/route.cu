// route.cu -- SVG-EAR's compensation-error probe and greedy error-to-cost
// routing under a density budget.
//
// Method: "SVG-EAR measured error" (frontier-cs.org blog), probe paragraph:
// one probe per query cluster (its mean query), scored against every real key
// of a block, summing |e^{s_bar} v_bar - e^{s_j} v_j|^2 over the block, the
// error divided by the block's token pairs; budget spent per query cluster.
// The pith.science review of the SVG-EAR paper ("What carries the argument"):
// greedy selection of the highest error-to-cost blocks under a density budget;
// the probe costs O(Cq * Nk * d).
//
// Kernels (fp32 throughout):
//   probe_rowmax  m_i = max_t scale*qbar_i.k_t, by an order-independent
//                 atomicMax on order-preserving integer keys (deterministic);
//   probe_error   one block per (key cluster, 32 probes, head): every probe
//                 against every key of the cluster, direct form of the error
//                 (no expansion, so small errors are not lost to cancellation);
//   route_select  one block per (query cluster, head): r_c = E/n_c, a bitonic
//                 sort on (r desc, c asc), the greedy take-if-fits scan, and
//                 an ascending list of the taken clusters;
//   route_compact one block per head: CSR offsets and the packed pair list.
#include "common.cuh"
#include "launchers.h"

namespace svgear {

constexpr int kPrProbes = 32;    // probes per block (one per lane)
constexpr int kPrKeys = 64;      // keys staged per step
constexpr int kPrThreads = 256;  // 8 warps, 8 keys each per step

template <int D> struct ProbeSmem {
    static constexpr int kPad = D + 4;   // float4-aligned rows, conflict-free
};

template <typename T, int D>
__global__ void __launch_bounds__(kPrThreads)
probe_rowmax_kernel(const float* __restrict__ qbar, int Cq, const T* __restrict__ Kp,
                    int Nk, float scale, uint32_t* __restrict__ rowmax) {
    constexpr int P = ProbeSmem<D>::kPad;
    constexpr int EPC = Elem<T>::kPerChunk;
    extern __shared__ __align__(16) float sm[];
    float* Qs = sm;                 // [32][P]
    float* Ks = Qs + kPrProbes * P; // [kPrKeys][P]
    const int bh = blockIdx.z, i0 = blockIdx.y * kPrProbes, tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    const int keys_per_block = kPrKeys * 4;
    const int t_begin = blockIdx.x * keys_per_block;
    for (int q = tid; q < kPrProbes * D; q += kPrThreads) {
        const int p = q / D, k = q % D;
        Qs[p * P + k] = (i0 + p < Cq) ? qbar[((size_t)bh * Cq + i0 + p) * D + k] : 0.f;
    }
    const T* Kh = Kp + (size_t)bh * Nk * D;
    float best = __int_as_float(0xff800000);
    for (int kb = 0; kb < 4; ++kb) {
        const int tb = t_begin + kb * kPrKeys;
        __syncthreads();
        for (int q = tid; q < kPrKeys * (D / EPC); q += kPrThreads) {
            const int r = q / (D / EPC), col = (q % (D / EPC)) * EPC;
            float v[EPC];
            if (tb + r < Nk) Elem<T>::load(Kh + (size_t)(tb + r) * D + col, v);
            else
#pragma unroll
                for (int e = 0; e < EPC; ++e) v[e] = 0.f;
#pragma unroll
            for (int e = 0; e < EPC; ++e) Ks[r * P + col + e] = v[e];
        }
        __syncthreads();
        float acc[8];
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) acc[jj] = 0.f;
        const float* qr = Qs + lane * P;
#pragma unroll 2
        for (int k = 0; k < D; k += 4) {
            const float4 qv = *reinterpret_cast<const float4*>(qr + k);
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                const float4 kv = *reinterpret_cast<const float4*>(Ks + (warp * 8 + jj) * P + k);
                acc[jj] = fmaf(qv.x, kv.x, acc[jj]);
                acc[jj] = fmaf(qv.y, kv.y, acc[jj]);
                acc[jj] = fmaf(qv.z, kv.z, acc[jj]);
                acc[jj] = fmaf(qv.w, kv.w, acc[jj]);
            }
        }
#pragma unroll
        for (int jj = 0; jj < 8; ++jj)
            if (tb + warp * 8 + jj < Nk) best = fmaxf(best, scale * acc[jj]);
    }
    if (i0 + lane < Cq)
        atomicMax(rowmax + (size_t)bh * Cq + i0 + lane, float_to_ordered(best));
}

// VF: the value-free error sum_t (a_ic - b_it)^2 (values not read).
template <typename T, int D, bool VF>
__global__ void __launch_bounds__(kPrThreads)
probe_error_kernel(const float* __restrict__ qbar, int Cq, const T* __restrict__ Kp,
                   const T* __restrict__ Vp, const float* __restrict__ kbar,
                   const float* __restrict__ vbar, const int32_t* __restrict__ k_off,
                   int Ck, int Nk, float scale, const uint32_t* __restrict__ rowmax,
                   float* __restrict__ E) {
    constexpr int P = ProbeSmem<D>::kPad;
    constexpr int EPC = Elem<T>::kPerChunk;
    extern __shared__ __align__(16) float sm[];
    float* Qs = sm;                    // [32][P] probes
    float* AV = Qs + kPrProbes * P;    // [32][P] a_ic * vbar_c
    float* Ks = AV + kPrProbes * P;    // [kPrKeys][P]
    float* Vs = Ks + kPrKeys * P;      // [kPrKeys][P]
    float* red = Vs + kPrKeys * P;     // [8][32]
    __shared__ float kb_s[D];
    const int c = blockIdx.x, i0 = blockIdx.y * kPrProbes, bh = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int32_t* off = k_off + (size_t)bh * (Ck + 1);
    const int a = off[c], b = off[c + 1];
    const int ip = i0 + lane;
    if (b <= a || a < 0 || b > Nk) {   // empty (or malformed) key cluster: no error
        if (warp == 0 && ip < Cq) E[((size_t)bh * Cq + ip) * Ck + c] = 0.f;
        return;
    }
    for (int q = tid; q < kPrProbes * D; q += kPrThreads) {
        const int p = q / D, k = q % D;
        Qs[p * P + k] = (i0 + p < Cq) ? qbar[((size_t)bh * Cq + i0 + p) * D + k] : 0.f;
    }
    for (int k = tid; k < D; k += kPrThreads) kb_s[k] = kbar[((size_t)bh * Ck + c) * D + k];
    __syncthreads();
    // a_ic = exp(scale * qbar_i . kbar_c - m_i), one lane per probe
    const float m = (ip < Cq) ? ordered_to_float(rowmax[(size_t)bh * Cq + ip]) : 0.f;
    float dotk = 0.f;
    for (int k = 0; k < D; ++k) dotk = fmaf(Qs[lane * P + k], kb_s[k], dotk);
    const float aic = expf(scale * dotk - m);
    // every thread needs a_ic of every probe: broadcast through smem
    if (warp == 0) red[lane] = aic;
    __syncthreads();
    if constexpr (!VF) {   // the value-free error reads no values
        const float* vb = vbar + ((size_t)bh * Ck + c) * D;
        for (int q = tid; q < kPrProbes * D; q += kPrThreads) {
            const int p = q / D, k = q % D;
            AV[p * P + k] = red[p] * vb[k];
        }
    }
    const T* Kh = Kp + (size_t)bh * Nk * D;
    const T* Vh = VF ? nullptr : Vp + (size_t)bh * Nk * D;
    float err = 0.f;
    for (int tb = a; tb < b; tb += kPrKeys) {
        __syncthreads();
        for (int q = tid; q < kPrKeys * (D / EPC); q += kPrThreads) {
            const int r = q / (D / EPC), col = (q % (D / EPC)) * EPC;
            float kv[EPC], vv[EPC];
            if (tb + r < b) {
                Elem<T>::load(Kh + (size_t)(tb + r) * D + col, kv);
                if constexpr (!VF) {
                    Elem<T>::load(Vh + (size_t)(tb + r) * D + col, vv);
                } else {
#pragma unroll
                    for (int e = 0; e < EPC; ++e) vv[e] = 0.f;
                }
            } else {
#pragma unroll
                for (int e = 0; e < EPC; ++e) { kv[e] = 0.f; vv[e] = 0.f; }
            }
#pragma unroll
            for (int e = 0; e < EPC; ++e) { Ks[r * P + col + e] = kv[e]; Vs[r * P + col + e] = vv[e]; }
        }
        __syncthreads();
        // scores of this lane's probe against the warp's 8 keys
        float s[8];
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) s[jj] = 0.f;
        const float* qr = Qs + lane * P;
#pragma unroll 2
        for (int k = 0; k < D; k += 4) {
            const float4 qv = *reinterpret_cast<const float4*>(qr + k);
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                const float4 kv = *reinterpret_cast<const float4*>(Ks + (warp * 8 + jj) * P + k);
                s[jj] = fmaf(qv.x, kv.x, s[jj]);
                s[jj] = fmaf(qv.y, kv.y, s[jj]);
                s[jj] = fmaf(qv.z, kv.z, s[jj]);
                s[jj] = fmaf(qv.w, kv.w, s[jj]);
            }
        }
        float bw[8];
#pragma unroll
        for (int jj = 0; jj < 8; ++jj)
            bw[jj] = (tb + warp * 8 + jj < b) ? expf(scale * s[jj] - m) : 0.f;
        if constexpr (VF) {   // value-free: (a - b)^2 per key
#pragma unroll
            for (int jj = 0; jj < 8; ++jj)
                if (tb + warp * 8 + jj < b) err += (aic - bw[jj]) * (aic - bw[jj]);
        } else {
            // direct form: sum_k (a vbar_k - b v_k)^2 per key
            float e8[8];
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) e8[jj] = 0.f;
            const float* avr = AV + lane * P;
#pragma unroll 2
            for (int k = 0; k < D; k += 4) {
                const float4 av = *reinterpret_cast<const float4*>(avr + k);
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                    const float4 vv = *reinterpret_cast<const float4*>(Vs + (warp * 8 + jj) * P + k);
                    float d0 = fmaf(-bw[jj], vv.x, av.x), d1 = fmaf(-bw[jj], vv.y, av.y);
                    float d2 = fmaf(-bw[jj], vv.z, av.z), d3 = fmaf(-bw[jj], vv.w, av.w);
                    e8[jj] = fmaf(d0, d0, e8[jj]);
                    e8[jj] = fmaf(d1, d1, e8[jj]);
                    e8[jj] = fmaf(d2, d2, e8[jj]);
                    e8[jj] = fmaf(d3, d3, e8[jj]);
                }
            }
#pragma unroll
            for (int jj = 0; jj < 8; ++jj)
                if (tb + warp * 8 + jj < b) err += e8[jj];
        }
    }
    __syncthreads();
    red[warp * 32 + lane] = err;
    __syncthreads();
    if (warp == 0 && ip < Cq) {
        float tot = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) tot += red[w * 32 + lane];
        E[((size_t)bh * Cq + ip) * Ck + c] = tot;
    }
}

__global__ void fill_u32_kernel(uint32_t* p, size_t n, uint32_t v) {
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (size_t)gridDim.x * blockDim.x)
        p[i] = v;
}

template <typename T, int D>
static int probe_impl(const float* qbar, int Cq, const void* Kp, const void* Vp,
                      const float* kbar, const float* vbar, const int32_t* k_off, int Ck,
                      svgear_dims kd, float scale, float* E, uint32_t* rowmax,
                      bool value_free, cudaStream_t st) {
    constexpr int P = ProbeSmem<D>::kPad;
    const int BH = kd.B * kd.H, Nk = kd.N;
    const size_t nrow = (size_t)BH * Cq;
    fill_u32_kernel<<<ceil_div((long long)nrow, 256) < 1024 ? ceil_div((long long)nrow, 256) : 1024,
                      256, 0, st>>>(rowmax, nrow, 0x007FFFFFu);  // ordered(-inf)
    const size_t sm1 = sizeof(float) * (kPrProbes + kPrKeys) * P;
    count_launches(1);
    if (cudaFuncSetAttribute(probe_rowmax_kernel<T, D>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm1) != cudaSuccess)
        return SVGEAR_ERR_CUDA;
    probe_rowmax_kernel<T, D><<<dim3(ceil_div(Nk, kPrKeys * 4), ceil_div(Cq, kPrProbes), BH),
                                kPrThreads, sm1, st>>>(qbar, Cq, static_cast<const T*>(Kp), Nk,
                                                       scale, rowmax);
    count_launches(1);
    const size_t sm2 = sizeof(float) * ((2 * kPrProbes + 2 * kPrKeys) * P + 8 * 32);
    auto kern = value_free ? probe_error_kernel<T, D, true> : probe_error_kernel<T, D, false>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm2) !=
        cudaSuccess)
        return SVGEAR_ERR_CUDA;
    kern<<<dim3(Ck, ceil_div(Cq, kPrProbes), BH), kPrThreads, sm2, st>>>(
        qbar, Cq, static_cast<const T*>(Kp), static_cast<const T*>(Vp), kbar, vbar, k_off, Ck,
        Nk, scale, rowmax, E);
    count_launches(1);
    SVGEAR_LAUNCH_CHECK();
    return SVGEAR_OK;
}

template <typename T, int D>
static int probe_disp(const float* qbar, int Cq, const void* Kp, const void* Vp,
                      const float* kbar, const float* vbar, const int32_t* k_off, int Ck,
                      svgear_dims kd, float scale, float* E, uint32_t* rowmax, bool vf,
                      cudaStream_t st) {
    return probe_impl<T, D>(qbar, Cq, Kp, Vp, kbar, vbar, k_off, Ck, kd, scale, E, rowmax, vf, st);
}

int launch_probe(const float* qbar, int Cq, const void* Kp, const void* Vp, const float* kbar,
                 const float* vbar, const int32_t* k_off, int Ck, svgear_dims kd, float scale,
                 float* E, uint32_t* rowmax, cudaStream_t st, bool value_free) {
    if (kd.dtype == SVGEAR_BF16) {
        if (kd.d == 128) return probe_disp<__nv_bfloat16, 128>(qbar, Cq, Kp, Vp, kbar, vbar, k_off, Ck, kd, scale, E, rowmax, value_free, st);
        if (kd.d == 64) return probe_disp<__nv_bfloat16, 64>(qbar, Cq, Kp, Vp, kbar, vbar, k_off, Ck, kd, scale, E, rowmax, value_free, st);
    } else if (kd.dtype == SVGEAR_F32) {
        if (kd.d == 128) return probe_disp<float, 128>(qbar, Cq, Kp, Vp, kbar, vbar, k_off, Ck, kd, scale, E, rowmax, value_free, st);
        if (kd.d == 64) return probe_disp<float, 64>(qbar, Cq, Kp, Vp, kbar, vbar, k_off, Ck, kd, scale, E, rowmax, value_free, st);
    }
    return SVGEAR_ERR_UNSUPPORTED;
}

// ---------------------------------------------------------------------------
// Routing.  Sort key (ascending): high word = ~ordered(r) (r descending), NaN
// -> 0xFFFFFFFE, empty cluster / padding -> 0xFFFFFFFF; low word = c.
// ---------------------------------------------------------------------------
constexpr int kRtThreads = 256;

__global__ void __launch_bounds__(kRtThreads)
route_select_kernel(const float* __restrict__ E, const int32_t* __restrict__ q_off, int Cq,
                    const int32_t* __restrict__ k_off, int Ck, long long budget_all,
                    const int32_t* __restrict__ budgets, int32_t* __restrict__ lists,
                    int32_t* __restrict__ counts) {
    extern __shared__ __align__(8) unsigned char smraw[];
    const int i = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    int P2 = 1;
    while (P2 < Ck) P2 <<= 1;
    unsigned long long* key = reinterpret_cast<unsigned long long*>(smraw);  // [P2]
    int32_t* nsz = reinterpret_cast<int32_t*>(key + P2);                    // [Ck]
    unsigned char* take = reinterpret_cast<unsigned char*>(nsz + Ck);        // [Ck]
    __shared__ int s_cnt[kRtThreads];
    const int32_t* qo = q_off + (size_t)bh * (Cq + 1);
    int32_t* list = lists + ((size_t)bh * Cq + i) * Ck;
    if (qo[i + 1] <= qo[i]) {
        if (tid == 0) counts[(size_t)bh * Cq + i] = 0;
        return;
    }
    const int32_t* ko = k_off + (size_t)bh * (Ck + 1);
    const float* Er = E + ((size_t)bh * Cq + i) * Ck;
    for (int c = tid; c < P2; c += kRtThreads) {
        unsigned long long kk = ~0ull;
        if (c < Ck) {
            const int n = ko[c + 1] - ko[c];
            nsz[c] = n;
            take[c] = 0;
            if (n > 0) {
                float r = __fdiv_rn(Er[c], (float)n);
                uint32_t hi;
                if (r != r) hi = 0xFFFFFFFEu;
                else {
                    if (r == 0.f) r = 0.f;   // -0 ranks with +0
                    hi = ~float_to_ordered(r);
                }
                kk = ((unsigned long long)hi << 32) | (uint32_t)c;
            }
        }
        key[c] = kk;
    }
    __syncthreads();
    // bitonic sort, ascending
    for (int k = 2; k <= P2; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int x = tid; x < P2; x += kRtThreads) {
                const int y = x ^ j;
                if (y > x) {
                    const unsigned long long a = key[x], b = key[y];
                    const bool up = (x & k) == 0;
                    if ((a > b) == up) { key[x] = b; key[y] = a; }
                }
            }
            __syncthreads();
        }
    }
    if (tid == 0) {
        const long long budget = budgets ? (long long)budgets[(size_t)bh * Cq + i] : budget_all;
        long long used = 0;
        for (int x = 0; x < Ck; ++x) {
            const unsigned long long kk = key[x];
            if ((kk >> 32) == 0xFFFFFFFFull) break;
            const int c = (int)(kk & 0xFFFFFFFFull);
            const int n = nsz[c];
            if (used + n <= budget) { take[c] = 1; used += n; }
        }
    }
    __syncthreads();
    // ascending compaction of the taken clusters
    const int per = (Ck + kRtThreads - 1) / kRtThreads;
    const int c0 = tid * per, c1 = min(Ck, c0 + per);
    int cnt = 0;
    for (int c = c0; c < c1; ++c) cnt += take[c];
    s_cnt[tid] = cnt;
    __syncthreads();
    if (tid == 0) {
        int run = 0;
        for (int t = 0; t < kRtThreads; ++t) { int v = s_cnt[t]; s_cnt[t] = run; run += v; }
        counts[(size_t)bh * Cq + i] = run;
    }
    __syncthreads();
    int w = s_cnt[tid];
    for (int c = c0; c < c1; ++c)
        if (take[c]) list[w++] = c;
}

__global__ void route_compact_kernel(const int32_t* __restrict__ lists,
                                     const int32_t* __restrict__ counts, int Cq, int Ck,
                                     int32_t* __restrict__ pair_off, int32_t* __restrict__ pair_kc) {
    extern __shared__ int32_t offs[];   // [Cq + 1]
    const int bh = blockIdx.x, tid = threadIdx.x;
    if (tid == 0) {
        int run = 0;
        for (int i = 0; i < Cq; ++i) { offs[i] = run; run += counts[(size_t)bh * Cq + i]; }
        offs[Cq] = run;
    }
    __syncthreads();
    int32_t* po = pair_off + (size_t)bh * (Cq + 1);
    for (int i = tid; i <= Cq; i += blockDim.x) po[i] = offs[i];
    int32_t* pk = pair_kc + (size_t)bh * Cq * Ck;
    for (int i = 0; i < Cq; ++i) {
        const int n = offs[i + 1] - offs[i];
        const int32_t* src = lists + ((size_t)bh * Cq + i) * Ck;
        for (int e = tid; e < n; e += blockDim.x) pk[offs[i] + e] = src[e];
    }
}

int launch_route_select(const float* E, const int32_t* q_off, int Cq, const int32_t* k_off,
                        int Ck, int BH, long long budget, const int32_t* budgets, int32_t* lists,
                        int32_t* counts, int32_t* pair_off, int32_t* pair_kc, cudaStream_t st) {
    int P2 = 1;
    while (P2 < Ck) P2 <<= 1;
    const size_t sm = sizeof(unsigned long long) * P2 + sizeof(int32_t) * Ck + Ck + 16;
    if (sm > 48 * 1024 &&
        cudaFuncSetAttribute(route_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)sm) != cudaSuccess)
        return SVGEAR_ERR_CUDA;
    route_select_kernel<<<dim3(Cq, BH), kRtThreads, sm, st>>>(E, q_off, Cq, k_off, Ck, budget,
                                                              budgets, lists, counts);
    count_launches(1);
    route_compact_kernel<<<BH, 256, sizeof(int32_t) * (Cq + 1), st>>>(lists, counts, Cq, Ck,
                                                                       pair_off, pair_kc);
    count_launches(1);
    SVGEAR_LAUNCH_CHECK();
    return SVGEAR_OK;
}


// ---------------------------------------------------------------------------
// Top-p budget (SVG2 summary, section 3.4, "From pre-softmax scores to
// attention probability estimates" and "Top-p selection for dynamic budget
// allocation"; SVG-EAR blog, budget paragraph): per query cluster i, the keys
// of the key clusters that hold p of the size-weighted centroid estimate
//   P'_ij = n_j e^{S_ij} / sum_l n_l e^{S_il},   S_ij = scale * qbar_i . kbar_j,
// taken in descending P' (ties: lower j) until the running sum reaches p.
// One block per (query cluster, head), in fp64 throughout: S (the centroids
// are fp32), w_j = n_j e^{S_ij - max S}, a bitonic sort of (w, j), and the
// running sum compared with p * sum(w), both summed in sorted order.  Empty
// key clusters and NaN scores take no part; an empty query cluster gets 0.
// ---------------------------------------------------------------------------
constexpr int kTpThreads = 256;

template <int D>
__global__ void __launch_bounds__(kTpThreads)
topp_budget_kernel(const float* __restrict__ qbar, const int32_t* __restrict__ q_off, int Cq,
                   const float* __restrict__ kbar, const int32_t* __restrict__ k_off, int Ck,
                   double p, double scale, int32_t* __restrict__ budget) {
    extern __shared__ __align__(8) unsigned char smraw[];
    __shared__ double q[D];
    __shared__ double red[kTpThreads / 32];
    const int i = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    int P2 = 1;
    while (P2 < Ck) P2 <<= 1;
    double* w = reinterpret_cast<double*>(smraw);          // [P2]
    int32_t* idx = reinterpret_cast<int32_t*>(w + P2);     // [P2]
    int32_t* nsz = idx + P2;                                // [Ck]
    const int32_t* qo = q_off + (size_t)bh * (Cq + 1);
    if (qo[i + 1] <= qo[i]) {
        if (tid == 0) budget[(size_t)bh * Cq + i] = 0;
        return;
    }
    const int32_t* ko = k_off + (size_t)bh * (Ck + 1);
    for (int k = tid; k < D; k += kTpThreads) q[k] = (double)qbar[((size_t)bh * Cq + i) * D + k];
    __syncthreads();
    double mx = -INFINITY;
    for (int c = tid; c < P2; c += kTpThreads) {
        double sc = NAN;
        if (c < Ck) {
            const int n = ko[c + 1] - ko[c];
            nsz[c] = n;
            if (n > 0) {
                const float* kr = kbar + ((size_t)bh * Ck + c) * D;
                double acc = 0.0;
                for (int k = 0; k < D; ++k) acc = fma(q[k], (double)kr[k], acc);
                sc = scale * acc;
                if (sc > mx) mx = sc;
            }
        }
        w[c] = sc;
        idx[c] = c;
    }
    // block max of the scores
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if ((tid & 31) == 0) red[tid >> 5] = mx;
    __syncthreads();
    if (tid == 0) {
        double m = red[0];
        for (int k = 1; k < kTpThreads / 32; ++k) m = fmax(m, red[k]);
        red[0] = m;
    }
    __syncthreads();
    const double smax = red[0];
    // weights; excluded entries get -1 and sort last
    for (int c = tid; c < P2; c += kTpThreads) {
        const double sc = w[c];
        w[c] = (c < Ck && sc == sc) ? (double)nsz[c] * exp(sc - smax) : -1.0;
    }
    __syncthreads();
    // bitonic sort: descending w, ties to the lower index
    for (int k = 2; k <= P2; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int x = tid; x < P2; x += kTpThreads) {
                const int y = x ^ j;
                if (y > x) {
                    const double wa = w[x], wb = w[y];
                    const int ia = idx[x], ib = idx[y];
                    const bool a_first = wa > wb || (wa == wb && ia < ib);
                    const bool up = (x & k) == 0;
                    if (a_first != up) {
                        w[x] = wb; w[y] = wa;
                        idx[x] = ib; idx[y] = ia;
                    }
                }
            }
            __syncthreads();
        }
    }
    if (tid == 0) {
        double total = 0.0;
        for (int x = 0; x < Ck && w[x] >= 0.0; ++x) total += w[x];
        const double target = p * total;
        double cum = 0.0;
        long long keys = 0;
        for (int x = 0; x < Ck && w[x] >= 0.0; ++x) {
            cum += w[x];
            keys += nsz[idx[x]];
            if (cum >= target) break;
        }
        budget[(size_t)bh * Cq + i] = (int32_t)keys;
    }
}

int launch_topp_budget(const float* qbar, const int32_t* q_off, int Cq, const float* kbar,
                       const int32_t* k_off, int Ck, int BH, int D, double p, double scale,
                       int32_t* budget, cudaStream_t st) {
    int P2 = 1;
    while (P2 < Ck) P2 <<= 1;
    const size_t sm = (sizeof(double) + sizeof(int32_t)) * P2 + sizeof(int32_t) * Ck + 16;
    if (D == 128) {
        if (sm > 48 * 1024 && cudaFuncSetAttribute(topp_budget_kernel<128>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   (int)sm) != cudaSuccess)
            return SVGEAR_ERR_CUDA;
        topp_budget_kernel<128><<<dim3(Cq, BH), kTpThreads, sm, st>>>(qbar, q_off, Cq, kbar, k_off,
                                                                      Ck, p, scale, budget);
    } else {
        if (sm > 48 * 1024 && cudaFuncSetAttribute(topp_budget_kernel<64>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   (int)sm) != cudaSuccess)
            return SVGEAR_ERR_CUDA;
        topp_budget_kernel<64><<<dim3(Cq, BH), kTpThreads, sm, st>>>(qbar, q_off, Cq, kbar, k_off,
                                                                     Ck, p, scale, budget);
    }
    count_launches(1);
    SVGEAR_LAUNCH_CHECK();
    return SVGEAR_OK;
}

}  // namespace svgear
