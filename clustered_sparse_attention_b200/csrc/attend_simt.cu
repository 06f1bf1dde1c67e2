// attend_simt.cu -- fp32 SIMT attention over the selected cluster blocks plus
// the centroid compensation of every skipped key cluster, in one online
// softmax; the fp32 path of svgear_attend (its 1e-5 tolerance rules out
// reduced-precision tensor-core operands).
//
// Method: "SVG-EAR measured error" (frontier-cs.org blog), toy example: a
// skipped cluster of n keys whose centroid scores s_bar weighs n e^{s_bar}
// and carries its mean value; the SVG-EAR task page (agent step 3): the
// skipped cluster acts as one key at its centroid with its score raised by
// log n, and each row goes straight back to its place in the video; SVG2
// summary section 3.4 (permutation validity): O = pi_q^T Attn(pi_q Q, pi_k K,
// pi_k V).
//
// One block per 64-row tile of one query cluster.  Keys of each selected
// cluster are staged 64 at a time; then the skipped, non-empty clusters'
// centroids are staged 64 at a time with a per-column bias log(n_c); with a
// key-variance table the score of a skipped cluster also gains
// var_coef * sum_k q_k^2 Var_c(k) (SVG-EAR blog, variance paragraph).
#include <math.h>

#include "common.cuh"
#include "launchers.h"

namespace svgear {

constexpr int kAtRows = 64, kAtKeys = 64, kAtThreads = 256;

template <typename T, int D>
__global__ void __launch_bounds__(kAtThreads)
attend_simt_kernel(const T* __restrict__ Qp, const T* __restrict__ Kp,
                   const T* __restrict__ Vp, int Nq, int Nk,
                   const int32_t* __restrict__ q_off, int Cq,
                   const int32_t* __restrict__ k_off, int Ck,
                   const int32_t* __restrict__ pair_off, const int32_t* __restrict__ pair_kc,
                   const float* __restrict__ kbar, const float* __restrict__ vbar,
                   const int32_t* __restrict__ q_perm, float scale, T* __restrict__ O,
                   const float* __restrict__ kvar, float var_coef) {
    constexpr int QP = D + 1;
    extern __shared__ __align__(16) float sm[];
    float* Qs = sm;                        // [64][D+1]
    float* Ks = Qs + kAtRows * QP;         // [64][D+1]
    float* Vs = Ks + kAtKeys * QP;         // [64][D]
    float* Ps = Vs + kAtKeys * D;          // [64][65]
    float* bias = Ps + kAtRows * 65;       // [64]
    int32_t* comp = reinterpret_cast<int32_t*>(bias + kAtKeys);   // [Ck]
    unsigned char* sel = reinterpret_cast<unsigned char*>(comp + Ck);  // [Ck]
    // [64][D+1]: var_coef * key variance of the compensation tile's clusters
    float* Ws = reinterpret_cast<float*>(sel + ((Ck + 15) & ~15));
    __shared__ int s_i, s_r0, s_r1, s_ncomp;

    const int bh = blockIdx.y, tid = threadIdx.x;
    const int32_t* qo = q_off + (size_t)bh * (Cq + 1);
    const int32_t* ko = k_off + (size_t)bh * (Ck + 1);
    if (tid == 0) {
        int acc = 0, g = blockIdx.x;
        s_i = -1;
        for (int i = 0; i < Cq; ++i) {
            if (qo[i] < 0 || qo[i + 1] > Nq) continue;   // malformed segment: skipped
            const int n = qo[i + 1] - qo[i];
            const int nt = (n + kAtRows - 1) / kAtRows;
            if (g < acc + nt) {
                s_i = i;
                s_r0 = qo[i] + (g - acc) * kAtRows;
                s_r1 = min(qo[i + 1], s_r0 + kAtRows);
                break;
            }
            acc += nt;
        }
    }
    __syncthreads();
    if (s_i < 0) return;
    const int i = s_i, r0 = s_r0, r1 = s_r1;

    for (int c = tid; c < Ck; c += kAtThreads) sel[c] = 0;
    __syncthreads();
    const int32_t* pk = pair_kc + (size_t)bh * Cq * Ck;
    const int32_t* po = pair_off + (size_t)bh * (Cq + 1);
    const int e0 = po[i], e1 = po[i + 1];
    for (int e = e0 + tid; e < e1; e += kAtThreads) {
        const int c = pk[e];
        if ((unsigned)c < (unsigned)Ck) sel[c] = 1;
    }
    __syncthreads();
    if (tid == 0) {
        int n = 0;
        for (int c = 0; c < Ck; ++c)
            if (!sel[c] && ko[c + 1] > ko[c] && ko[c] >= 0 && ko[c + 1] <= Nk) comp[n++] = c;
        s_ncomp = n;
    }
    // query tile
    const T* Qh = Qp + (size_t)bh * Nq * D;
    for (int q = tid; q < kAtRows * D; q += kAtThreads) {
        const int r = q / D, k = q % D;
        Qs[r * QP + k] = (r0 + r < r1) ? Elem<T>::from(Qh[(size_t)(r0 + r) * D + k]) : 0.f;
    }
    __syncthreads();

    const int row = tid >> 2, sub = tid & 3;
    constexpr int OC = D / 4;
    float o[OC];
#pragma unroll
    for (int e = 0; e < OC; ++e) o[e] = 0.f;
    float m_run = -INFINITY, l_run = 0.f;

    const T* Kh = Kp + (size_t)bh * Nk * D;
    const T* Vh = Vp + (size_t)bh * Nk * D;
    const float* kbh = kbar + (size_t)bh * Ck * D;
    const float* vbh = vbar + (size_t)bh * Ck * D;

    auto process = [&](int nvalid, bool with_var) {
        // scores of row `row` against keys sub + 4m
        float s[16];
        float cmax = -INFINITY;
#pragma unroll
        for (int mm = 0; mm < 16; ++mm) {
            const int j = sub + 4 * mm;
            float acc = 0.f;
            const float* qr = Qs + row * QP;
            const float* kr = Ks + j * QP;
#pragma unroll 8
            for (int k = 0; k < D; ++k) acc = fmaf(qr[k], kr[k], acc);
            if (with_var) {   // + var_coef * sum_k q_k^2 Var_c(k)
                const float* wr = Ws + j * QP;
                float vacc = 0.f;
#pragma unroll 8
                for (int k = 0; k < D; ++k) vacc = fmaf(qr[k] * qr[k], wr[k], vacc);
                s[mm] = (j < nvalid) ? fmaf(acc, scale, vacc + bias[j]) : -INFINITY;
            } else {
                s[mm] = (j < nvalid) ? fmaf(acc, scale, bias[j]) : -INFINITY;
            }
            cmax = fmaxf(cmax, s[mm]);
        }
        cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, 1));
        cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, 2));
        const float m_new = fmaxf(m_run, cmax);
        const float alpha = (m_run == -INFINITY) ? 0.f : expf(m_run - m_new);
        float psum = 0.f;
#pragma unroll
        for (int mm = 0; mm < 16; ++mm) {
            const float p = (s[mm] == -INFINITY) ? 0.f : expf(s[mm] - m_new);
            Ps[row * 65 + sub + 4 * mm] = p;
            psum += p;
        }
        psum += __shfl_xor_sync(0xffffffffu, psum, 1);
        psum += __shfl_xor_sync(0xffffffffu, psum, 2);
        l_run = l_run * alpha + psum;
        m_run = m_new;
#pragma unroll
        for (int e = 0; e < OC; ++e) o[e] *= alpha;
        __syncthreads();
        for (int j = 0; j < nvalid; ++j) {
            const float p = Ps[row * 65 + j];
            const float* vr = Vs + j * D;
#pragma unroll
            for (int e = 0; e < OC; ++e) o[e] = fmaf(p, vr[sub + 4 * e], o[e]);
        }
        __syncthreads();
    };

    // exact part: every key of every selected cluster (ascending cluster id)
    for (int e = e0; e < e1; ++e) {
        const int c = pk[e];
        if ((unsigned)c >= (unsigned)Ck || ko[c] < 0 || ko[c + 1] > Nk) continue;
        for (int t0 = ko[c]; t0 < ko[c + 1]; t0 += kAtKeys) {
            const int nv = min(kAtKeys, ko[c + 1] - t0);
            for (int q = tid; q < kAtKeys * D; q += kAtThreads) {
                const int j = q / D, k = q % D;
                float kv = 0.f, vv = 0.f;
                if (j < nv) {
                    kv = Elem<T>::from(Kh[(size_t)(t0 + j) * D + k]);
                    vv = Elem<T>::from(Vh[(size_t)(t0 + j) * D + k]);
                }
                Ks[j * QP + k] = kv;
                Vs[j * D + k] = vv;
            }
            if (tid < kAtKeys) bias[tid] = 0.f;
            __syncthreads();
            process(nv, false);
        }
    }
    // compensation: each skipped non-empty cluster as one key at its centroid
    const int ncomp = s_ncomp;
    for (int b0 = 0; b0 < ncomp; b0 += kAtKeys) {
        const int nv = min(kAtKeys, ncomp - b0);
        for (int q = tid; q < kAtKeys * D; q += kAtThreads) {
            const int j = q / D, k = q % D;
            float kv = 0.f, vv = 0.f;
            if (j < nv) {
                const int c = comp[b0 + j];
                kv = kbh[(size_t)c * D + k];
                vv = vbh[(size_t)c * D + k];
            }
            Ks[j * QP + k] = kv;
            Vs[j * D + k] = vv;
            if (kvar) Ws[j * QP + k] = (j < nv) ? var_coef * kvar[((size_t)bh * Ck + comp[b0 + j]) * D + k] : 0.f;
        }
        if (tid < kAtKeys) {
            float bv = 0.f;
            if (tid < nv) {
                const int c = comp[b0 + tid];
                bv = logf((float)(ko[c + 1] - ko[c]));
            }
            bias[tid] = bv;
        }
        __syncthreads();
        process(nv, kvar != nullptr);
    }
    // epilogue: O[q_perm[p]] = num / den
    const int p = r0 + row;
    if (p < r1) {
        const int dst = q_perm[(size_t)bh * Nq + p];
        if ((unsigned)dst < (unsigned)Nq) {
            const float inv = 1.f / l_run;
            T* orow = O + ((size_t)bh * Nq + dst) * D;
#pragma unroll
            for (int e = 0; e < OC; ++e) orow[sub + 4 * e] = Elem<T>::to(o[e] * inv);
        }
    }
}

template <typename T, int D>
static int attend_simt_impl(const void* Qp, const void* Kp, const void* Vp, svgear_dims qd,
                            int Nk, const int32_t* q_off, int Cq, const int32_t* k_off, int Ck,
                            const int32_t* pair_off, const int32_t* pair_kc, const float* kbar,
                            const float* vbar, const int32_t* q_perm, float scale, void* O,
                            const float* kvar, float var_coef, cudaStream_t st) {
    constexpr int QP = D + 1;
    const size_t sm = sizeof(float) * (kAtRows * QP + kAtKeys * QP + kAtKeys * D + kAtRows * 65 +
                                       kAtKeys) +
                      sizeof(int32_t) * Ck + ((Ck + 15) & ~15) +
                      (kvar ? sizeof(float) * kAtKeys * QP : 0);
    if (cudaFuncSetAttribute(attend_simt_kernel<T, D>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm) != cudaSuccess)
        return SVGEAR_ERR_CUDA;
    const int BH = qd.B * qd.H;
    const int tiles = ceil_div(qd.N, kAtRows) + Cq;   // upper bound over ragged clusters
    attend_simt_kernel<T, D><<<dim3(tiles, BH), kAtThreads, sm, st>>>(
        static_cast<const T*>(Qp), static_cast<const T*>(Kp), static_cast<const T*>(Vp), qd.N,
        Nk, q_off, Cq, k_off, Ck, pair_off, pair_kc, kbar, vbar, q_perm, scale,
        static_cast<T*>(O), kvar, var_coef);
    count_launches(1);
    SVGEAR_LAUNCH_CHECK();
    return SVGEAR_OK;
}

int launch_attend_simt(const void* Qp, const void* Kp, const void* Vp, svgear_dims qd, int Nk,
                       const int32_t* q_off, int Cq, const int32_t* k_off, int Ck,
                       const int32_t* pair_off, const int32_t* pair_kc, const float* kbar,
                       const float* vbar, const int32_t* q_perm, float scale, void* O,
                       const float* kvar, float var_coef, cudaStream_t st) {
#define SVGEAR_AT(T, D)                                                                    \
    return attend_simt_impl<T, D>(Qp, Kp, Vp, qd, Nk, q_off, Cq, k_off, Ck, pair_off,       \
                                  pair_kc, kbar, vbar, q_perm, scale, O, kvar, var_coef, st)
    if (qd.dtype == SVGEAR_BF16) {
        if (qd.d == 128) SVGEAR_AT(__nv_bfloat16, 128);
        if (qd.d == 64) SVGEAR_AT(__nv_bfloat16, 64);
    } else if (qd.dtype == SVGEAR_F32) {
        if (qd.d == 128) SVGEAR_AT(float, 128);
        if (qd.d == 64) SVGEAR_AT(float, 64);
    }
#undef SVGEAR_AT
    return SVGEAR_ERR_UNSUPPORTED;
}

}  // namespace svgear
