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
//   probe_error   one block per (key cluster, 128 probes, head): every probe
//                 against every key of the cluster, the error expanded around
//                 the key's residual from its cluster's value mean (see the
//                 register-tiled section below), shifted by the cluster's own
//                 maximum score m_ic and summed in a fixed order;
//   probe_rescale one warp per probe row: m_i = max_c m_ic (the maximum over
//                 every key of the head) and E_ic <- E_ic e^{2 (m_ic - m_i)};
//   route_select  one block per (query cluster, head): r_c = E/n_c, a bitonic
//                 sort on (r desc, c asc), the greedy take-if-fits scan, and
//                 an ascending list of the taken clusters;
//   route_compact one block per head: CSR offsets and the packed pair list.
#include "common.cuh"
#include "launchers.h"

namespace svgear {

// ---------------------------------------------------------------------------
// Probe, register-tiled: a block of up to 128 probes against a tile of 64
// keys, each thread 8 probes x 8 keys (probes 4pi..4pi+3 and 64+4pi..,
// keys 4ki..4ki+3 and 32+4ki.., so both shared-memory reads are free of
// bank conflicts).  Scores accumulate over k in order, like the plain form.
// The error of key t (cluster c, residual w_t = v_t - vbar_c) is evaluated
// as (a-b)^2 |vbar_c|^2 - 2 (a-b) b vbar_c.w_t + b^2 |w_t|^2 -- the same
// quantity as |a vbar_c - b v_t|^2 -- so a (probe, key) pair costs its score
// and a handful of scalar operations; vbar_c.w_t and |w_t|^2 come once per
// key from the cluster's value rows.
// ---------------------------------------------------------------------------
constexpr int kPbP = 128;        // probes per block
constexpr int kPbK = 64;         // keys per tile
constexpr int kPbThreads = 128;
static_assert(kPbThreads == kPbP, "one thread per probe of a block (the centroid scores)");

// qT[bh][blk][k][p] = qbar[bh][blk * 128 + p][k] (0 past Cq)
template <int D>
__global__ void probe_qT_kernel(const float* __restrict__ qbar, int Cq, int nPB,
                                float* __restrict__ qT) {
    const int blk = blockIdx.x, bh = blockIdx.y;
    float* out = qT + ((size_t)bh * nPB + blk) * D * kPbP;
    for (int e = threadIdx.x; e < D * kPbP; e += blockDim.x) {
        const int k = e / kPbP, p = e % kPbP, i = blk * kPbP + p;
        out[e] = i < Cq ? qbar[((size_t)bh * Cq + i) * D + k] : 0.f;
    }
}

template <int D>
__device__ __forceinline__ void pb_load_q(const float* __restrict__ qT, float* Qs) {
    const float4* src = reinterpret_cast<const float4*>(qT);
    float4* dst = reinterpret_cast<float4*>(Qs);
    for (int e = threadIdx.x; e < D * kPbP / 4; e += kPbThreads) dst[e] = __ldg(src + e);
}

// Ks[k][t] = key t0 + t, dimension k (0 past t_end)
template <typename T, int D>
__device__ __forceinline__ void pb_load_k(const T* __restrict__ Kh, int t0, int t_end, float* Ks) {
    constexpr int EPC = Elem<T>::kPerChunk;
    constexpr int NCH = D / EPC;
    for (int idx = threadIdx.x; idx < kPbK * NCH; idx += kPbThreads) {
        const int t = idx % kPbK, ch = idx / kPbK;
        float x[EPC];
        if (t0 + t < t_end) {
            Elem<T>::unpack(Elem<T>::load_raw(Kh + (size_t)(t0 + t) * D + ch * EPC), x);
        } else {
#pragma unroll
            for (int e = 0; e < EPC; ++e) x[e] = 0.f;
        }
#pragma unroll
        for (int e = 0; e < EPC; ++e) Ks[(ch * EPC + e) * kPbK + t] = x[e];
    }
}

// NJ = 8: all of the thread's keys; NJ = 4: only keys 4ki..4ki+3 (a tile with
// at most 32 keys, whose upper half is padding).  NI likewise for the probes:
// NI = 4 takes only probes 4pi..4pi+3 (a probe block with at most 64 probes).
// Skipped entries stay zero.
template <int D, int NI, int NJ>
__device__ __forceinline__ void pb_scores(const float* Qs, const float* Ks, int pi, int ki,
                                          float (&acc)[8][8]) {
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
#pragma unroll 2
    for (int k = 0; k < D; ++k) {
        const float4 qa = *reinterpret_cast<const float4*>(Qs + k * kPbP + pi * 4);
        float4 qb = make_float4(0.f, 0.f, 0.f, 0.f);
        if (NI == 8) qb = *reinterpret_cast<const float4*>(Qs + k * kPbP + 64 + pi * 4);
        const float4 ka = *reinterpret_cast<const float4*>(Ks + k * kPbK + ki * 4);
        float4 kb = make_float4(0.f, 0.f, 0.f, 0.f);
        if (NJ == 8) kb = *reinterpret_cast<const float4*>(Ks + k * kPbK + 32 + ki * 4);
        const float q[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
        const float kk[8] = {ka.x, ka.y, ka.z, ka.w, kb.x, kb.y, kb.z, kb.w};
#pragma unroll
        for (int i = 0; i < NI; ++i)
#pragma unroll
            for (int j = 0; j < NJ; ++j) acc[i][j] = fmaf(q[i], kk[j], acc[i][j]);
    }
}
__device__ __forceinline__ int pb_probe(int pi, int i) { return pi * 4 + (i & 3) + (i >> 2) * 64; }
__device__ __forceinline__ int pb_key(int ki, int j) { return ki * 4 + (j & 3) + (j >> 2) * 32; }

// E[bh][i][c] for the block's probes, one CTA per (key cluster c, probe
// block, head).  VF: the value-free error sum_t (a - b)^2.
template <typename T, int D, bool VF>
__global__ void __launch_bounds__(kPbThreads, 2)
probe_error_v2_kernel(const float* __restrict__ qT, int Cq, int nPB, const T* __restrict__ Kp,
                      const T* __restrict__ Vp, const float* __restrict__ kbar,
                      const float* __restrict__ vbar, const int32_t* __restrict__ k_off, int Ck,
                      int Nk, float scale, float* __restrict__ mloc,
                      float* __restrict__ E) {
    extern __shared__ __align__(16) float pbs[];
    float* Qs = pbs;                 // [D][128]
    float* Ks = Qs + D * kPbP;       // [D][64]
    float* red = Ks + D * kPbK;      // [4][128]
    float* kb = red + 4 * kPbP;      // [D] kbar_c
    float* vb = kb + D;              // [D] vbar_c
    float* al = vb + D;              // [64] vbar_c . w_t
    float* be = al + kPbK;           // [64] |w_t|^2
    const int c = blockIdx.x, blk = blockIdx.y, bh = blockIdx.z, tid = threadIdx.x;
    const int pi = tid & 15, ki = tid >> 4, lane = tid & 31, warp = tid >> 5;
    // the last probe block holds at most 64 probes: probes 64.. of the block
    // (the upper four of each thread's eight) are padding
    const bool half = Cq - blk * kPbP <= kPbP / 2;
    const int32_t* off = k_off + (size_t)bh * (Ck + 1);
    const int a0 = off[c], a1 = off[c + 1];
    if (a1 <= a0 || a0 < 0 || a1 > Nk) {   // empty (or malformed) key cluster: no error
        const int p = blk * kPbP + tid;
        if (p < Cq) {
            E[((size_t)bh * Cq + p) * Ck + c] = 0.f;
            mloc[((size_t)bh * Cq + p) * Ck + c] = -INFINITY;
        }
        return;
    }
    pb_load_q<D>(qT + ((size_t)bh * nPB + blk) * D * kPbP, Qs);
    for (int k = tid; k < D; k += kPbThreads) {
        kb[k] = kbar[((size_t)bh * Ck + c) * D + k];
        if (!VF) vb[k] = vbar[((size_t)bh * Ck + c) * D + k];
    }
    __syncthreads();
    // Every thread shifts its own keys' terms by its running maximum m_i of
    // the probe's scores (a rescale of its partial sum whenever a tile
    // raises it); the partial sums are brought to the cluster's maximum m_ic
    // before they are added, and a last kernel brings E to the row maximum
    // m_i = max_c m_ic: E(m) = e^{2 (m' - m)} E(m'), every term being
    // quadratic in (e^{sbar - m}, e^{s - m}).
    // the centroid's score of every probe, once per probe (thread p takes
    // probe p; the same sequential sum as the plain form), read back by the
    // eight threads that share each probe
    {
        float dotk = 0.f;
        for (int k = 0; k < D; ++k) dotk = fmaf(Qs[k * kPbP + tid], kb[k], dotk);
        red[tid] = scale * dotk;
    }
    __syncthreads();
    float ai[8], mi[8], sbar[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        sbar[i] = red[pb_probe(pi, i)];
        mi[i] = sbar[i];   // the centroid's score (the mean of the members' scores) starts it
        ai[i] = 1.f;
    }
    float gamma = 0.f;
    if (!VF)
        for (int k = 0; k < D; ++k) gamma = fmaf(vb[k], vb[k], gamma);
    const T* Kh = Kp + (size_t)bh * Nk * D;
    const T* Vh = VF ? nullptr : Vp + (size_t)bh * Nk * D;
    float err[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) err[i] = 0.f;
    for (int t0 = a0; t0 < a1; t0 += kPbK) {
        __syncthreads();
        pb_load_k<T, D>(Kh, t0, a1, Ks);
        if constexpr (!VF) {
            // per key: alpha = vbar_c . w, beta = |w|^2, two threads per key
            constexpr int EPC = Elem<T>::kPerChunk;
            const int t = tid >> 1, half = tid & 1;
            float sa = 0.f, sb = 0.f;
            if (t0 + t < a1) {
                const T* vr = Vh + (size_t)(t0 + t) * D + half * (D / 2);
#pragma unroll 4
                for (int ch = 0; ch < D / 2 / EPC; ++ch) {
                    float x[EPC];
                    Elem<T>::unpack(Elem<T>::load_raw(vr + ch * EPC), x);
#pragma unroll
                    for (int e = 0; e < EPC; ++e) {
                        const int k = half * (D / 2) + ch * EPC + e;
                        const float w = x[e] - vb[k];
                        sa = fmaf(vb[k], w, sa);
                        sb = fmaf(w, w, sb);
                    }
                }
            }
            sa += __shfl_xor_sync(0xffffffffu, sa, 1);
            sb += __shfl_xor_sync(0xffffffffu, sb, 1);
            if (half == 0) {
                al[t] = sa;
                be[t] = sb;
            }
        }
        __syncthreads();
        float acc[8][8];
        const bool tail = a1 - t0 <= kPbK / 2;   // a tail of at most 32 keys
        if (half)
            tail ? pb_scores<D, 4, 4>(Qs, Ks, pi, ki, acc) : pb_scores<D, 4, 8>(Qs, Ks, pi, ki, acc);
        else
            tail ? pb_scores<D, 8, 4>(Qs, Ks, pi, ki, acc) : pb_scores<D, 8, 8>(Qs, Ks, pi, ki, acc);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            float tmx = -INFINITY;
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (t0 + pb_key(ki, j) < a1) tmx = fmaxf(tmx, scale * acc[i][j]);
            if (tmx > mi[i]) {   // the shift grows: rescale what is summed so far
                err[i] *= expf(2.f * (mi[i] - tmx));
                mi[i] = tmx;
                ai[i] = expf(sbar[i] - tmx);
            }
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int tj = pb_key(ki, j);
            if (t0 + tj >= a1) continue;
            float alj = 0.f, bej = 0.f;
            if (!VF) {
                alj = al[tj];
                bej = be[tj];
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                if (half && i >= 4) continue;   // padding probes of a half block
                const float b = expf(scale * acc[i][j] - mi[i]);
                const float dab = ai[i] - b;
                if (VF) {
                    err[i] = fmaf(dab, dab, err[i]);
                } else {
                    const float e = fmaf(b * b, bej, fmaf(dab * dab, gamma, -2.f * dab * b * alj));
                    err[i] += e;
                }
            }
        }
    }
    // the cluster's maximum m_ic per probe: over the 8 threads of each probe
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float o = __shfl_xor_sync(0xffffffffu, mi[i], 16);
        const float eo = __shfl_xor_sync(0xffffffffu, err[i], 16);
        const float m2 = fmaxf(mi[i], o);
        err[i] = err[i] * expf(2.f * (mi[i] - m2)) + eo * expf(2.f * (o - m2));
        mi[i] = m2;
    }
    __syncthreads();
    float* redm = kb;   // kbar_c is no longer needed: the warps' maxima
    if (lane < 16)
#pragma unroll
        for (int i = 0; i < 8; ++i) red[warp * kPbP + pb_probe(pi, i)] = mi[i];
    __syncthreads();
    float mw[4];
    if (tid < kPbP) {
#pragma unroll
        for (int w = 0; w < 4; ++w) mw[w] = red[w * kPbP + tid];
    }
    __syncthreads();
    if (lane < 16)
#pragma unroll
        for (int i = 0; i < 8; ++i) red[warp * kPbP + pb_probe(pi, i)] = err[i];
    __syncthreads();
    (void)redm;
    const int p = blk * kPbP + tid;
    if (p < Cq) {
        const float m = fmaxf(fmaxf(mw[0], mw[1]), fmaxf(mw[2], mw[3]));
        float e = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w)
            e += red[w * kPbP + tid] * expf(2.f * (mw[w] - m));
        E[((size_t)bh * Cq + p) * Ck + c] = e;
        mloc[((size_t)bh * Cq + p) * Ck + c] = m;
    }
}

// E_ic <- E_ic e^{2 (m_ic - m_i)} with m_i = max_c m_ic (the maximum over
// every key of the head: each m_ic is the maximum over cluster c's keys),
// one warp per probe row; empty clusters (E = 0, m = -inf) stay 0.
__global__ void probe_rescale_kernel(float* __restrict__ E, const float* __restrict__ mloc, int Ck,
                                     long long rows) {
    const long long row = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const float* ml = mloc + row * Ck;
    float* er = E + row * Ck;
    float m = -INFINITY;
    for (int c = lane; c < Ck; c += 32) m = fmaxf(m, ml[c]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    for (int c = lane; c < Ck; c += 32) {
        const float mc = ml[c];
        er[c] = mc > -INFINITY ? er[c] * expf(2.f * (mc - m)) : 0.f;
    }
}

template <typename T, int D>
static int probe_impl(const float* qbar, int Cq, const void* Kp, const void* Vp,
                      const float* kbar, const float* vbar, const int32_t* k_off, int Ck,
                      svgear_dims kd, float scale, float* E, float* cmax, float* qT,
                      bool value_free, cudaStream_t st) {
    const int BH = kd.B * kd.H, Nk = kd.N;
    const int nPB = ceil_div(Cq, kPbP);
    const size_t nrow = (size_t)BH * Cq;
    probe_qT_kernel<D><<<dim3(nPB, BH), 256, 0, st>>>(qbar, Cq, nPB, qT);
    count_launches(1);
    const size_t sm1 = sizeof(float) * ((size_t)D * (kPbP + kPbK) + 4 * kPbP);
    const size_t sm2 = sm1 + sizeof(float) * (2 * D + 2 * kPbK);
    auto kern = value_free ? probe_error_v2_kernel<T, D, true> : probe_error_v2_kernel<T, D, false>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm2) !=
        cudaSuccess)
        return SVGEAR_ERR_CUDA;
    float* mloc = cmax;   // [BH][Cq][Ck]: m_ic, the maximum score of probe i over cluster c
    kern<<<dim3(Ck, nPB, BH), kPbThreads, sm2, st>>>(
        qT, Cq, nPB, static_cast<const T*>(Kp), static_cast<const T*>(Vp), kbar, vbar, k_off, Ck,
        Nk, scale, mloc, E);
    probe_rescale_kernel<<<(unsigned)ceil_div((long long)nrow, 8), 256, 0, st>>>(E, mloc, Ck,
                                                                                (long long)nrow);
    count_launches(2);
    SVGEAR_LAUNCH_CHECK();
    return SVGEAR_OK;
}

int launch_probe(const float* qbar, int Cq, const void* Kp, const void* Vp, const float* kbar,
                 const float* vbar, const int32_t* k_off, int Ck, svgear_dims kd, float scale,
                 float* E, float* cmax, float* qT, cudaStream_t st, bool value_free) {
    if (kd.dtype == SVGEAR_BF16) {
        if (kd.d == 128) return probe_impl<__nv_bfloat16, 128>(qbar, Cq, Kp, Vp, kbar, vbar, k_off, Ck, kd, scale, E, cmax, qT, value_free, st);
        if (kd.d == 64) return probe_impl<__nv_bfloat16, 64>(qbar, Cq, Kp, Vp, kbar, vbar, k_off, Ck, kd, scale, E, cmax, qT, value_free, st);
    } else if (kd.dtype == SVGEAR_F32) {
        if (kd.d == 128) return probe_impl<float, 128>(qbar, Cq, Kp, Vp, kbar, vbar, k_off, Ck, kd, scale, E, cmax, qT, value_free, st);
        if (kd.d == 64) return probe_impl<float, 64>(qbar, Cq, Kp, Vp, kbar, vbar, k_off, Ck, kd, scale, E, cmax, qT, value_free, st);
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
