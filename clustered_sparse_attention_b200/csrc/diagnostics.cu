// diagnostics.cu -- how close the sparse layer is to dense attention, on
// sampled query rows.
//
// Method: SVG2 summary, section 3.1 ("The oracle policy"): attention recall,
// the share of the original attention mass that the computed tokens keep;
// SVG-EAR review (pith.science), Fig. 6a: the attention MSE of the sparse
// output against full attention.  For query row p (permuted position) of
// query cluster i:
//   recall = sum_{u in the selected key clusters of i} e^{s_pu} / sum_u e^{s_pu}
//   err2   = | O_sparse[q_perm[p]] - O_dense(p) |^2,   ref2 = | O_dense(p) |^2
// with O_dense(p) = softmax over every key.  Not part of the layer: a
// measurement of it.
//
// B200 design: one CTA per sampled row; each of 8 warps streams every 8th key
// (a lane holds d/32 coordinates: one 32-lane dot product per key) with its
// own online softmax state, and the warps' states are merged at the end.
#include <math.h>

#include "common.cuh"
#include "launchers.h"

namespace svgear {

constexpr int kDgThreads = 256;
constexpr int kDgWarps = kDgThreads / 32;

template <typename T, int D>
__global__ void __launch_bounds__(kDgThreads)
diagnostics_kernel(const T* __restrict__ Qp, const T* __restrict__ Kp, const T* __restrict__ Vp,
                   int Nq, int Nk, const int32_t* __restrict__ q_off, int Cq,
                   const int32_t* __restrict__ k_off, int Ck, const int32_t* __restrict__ pair_off,
                   const int32_t* __restrict__ pair_kc, const T* __restrict__ O,
                   const int32_t* __restrict__ q_perm, float scale, const int32_t* __restrict__ rows,
                   int R, float* __restrict__ recall, float* __restrict__ err2,
                   float* __restrict__ ref2) {
    constexpr int EPL = D / 32;
    extern __shared__ unsigned char sel[];   // [Ck]: selected key clusters of the row's cluster
    __shared__ float q[D];
    __shared__ float wm[kDgWarps], wz[kDgWarps], wzs[kDgWarps];
    __shared__ float wo[kDgWarps][D];
    __shared__ float red[2][kDgWarps];
    __shared__ int s_i;
    const int r = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const size_t orow = (size_t)bh * R + r;
    const int p = rows[orow];
    const int32_t* qo = q_off + (size_t)bh * (Cq + 1);
    const int32_t* ko = k_off + (size_t)bh * (Ck + 1);
    if ((unsigned)p >= (unsigned)Nq) {
        if (tid == 0) recall[orow] = err2[orow] = ref2[orow] = NAN;
        return;
    }
    if (tid == 0) {
        int i = -1;
        for (int c = 0; c < Cq; ++c)
            if (qo[c] <= p && p < qo[c + 1]) { i = c; break; }
        s_i = i;
    }
    for (int c = tid; c < Ck; c += kDgThreads) sel[c] = 0;
    const T* Qh = Qp + (size_t)bh * Nq * D;
    for (int k = tid; k < D; k += kDgThreads) q[k] = Elem<T>::from(Qh[(size_t)p * D + k]);
    __syncthreads();
    const int i = s_i;
    if (i >= 0) {
        const int32_t* po = pair_off + (size_t)bh * (Cq + 1);
        const int32_t* pk = pair_kc + (size_t)bh * Cq * Ck;
        for (int e = po[i] + tid; e < po[i + 1]; e += kDgThreads) {
            const int c = pk[e];
            if ((unsigned)c < (unsigned)Ck) sel[c] = 1;
        }
    }
    __syncthreads();

    const T* Kh = Kp + (size_t)bh * Nk * D;
    const T* Vh = Vp + (size_t)bh * Nk * D;
    float qr[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) qr[e] = q[lane * EPL + e];
    float m = -INFINITY, Z = 0.f, Zs = 0.f, o[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) o[e] = 0.f;
    int c = 0;   // key cluster of key u (keys are visited in increasing order)
    for (int u = warp; u < Nk; u += kDgWarps) {
        while (c < Ck && ko[c + 1] <= u) ++c;
        const T* kr = Kh + (size_t)u * D + lane * EPL;
        float part = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) part = fmaf(qr[e], Elem<T>::from(kr[e]), part);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
        const float s = part * scale;
        if (s > m) {
            const float f = (m == -INFINITY) ? 0.f : expf(m - s);
            Z *= f;
            Zs *= f;
#pragma unroll
            for (int e = 0; e < EPL; ++e) o[e] *= f;
            m = s;
        }
        const float w = expf(s - m);
        Z += w;
        if (c < Ck && sel[c]) Zs += w;
        const T* vr = Vh + (size_t)u * D + lane * EPL;
#pragma unroll
        for (int e = 0; e < EPL; ++e) o[e] = fmaf(w, Elem<T>::from(vr[e]), o[e]);
    }
    if (lane == 0) {
        wm[warp] = m;
        wz[warp] = Z;
        wzs[warp] = Zs;
    }
#pragma unroll
    for (int e = 0; e < EPL; ++e) wo[warp][lane * EPL + e] = o[e];
    __syncthreads();
    // merge the warps' softmax states
    float M = -INFINITY;
    for (int w = 0; w < kDgWarps; ++w) M = fmaxf(M, wm[w]);
    float Zt = 0.f, Zst = 0.f;
    for (int w = 0; w < kDgWarps; ++w) {
        const float f = (wm[w] == -INFINITY) ? 0.f : expf(wm[w] - M);
        Zt += wz[w] * f;
        Zst += wzs[w] * f;
    }
    float e2 = 0.f, r2 = 0.f;
    if (tid < D) {
        float od = 0.f;
        for (int w = 0; w < kDgWarps; ++w) {
            const float f = (wm[w] == -INFINITY) ? 0.f : expf(wm[w] - M);
            od = fmaf(wo[w][tid], f, od);
        }
        od /= Zt;
        const int dst = q_perm[(size_t)bh * Nq + p];
        const float os = ((unsigned)dst < (unsigned)Nq)
                             ? Elem<T>::from(O[((size_t)bh * Nq + dst) * D + tid]) : NAN;
        e2 = (os - od) * (os - od);
        r2 = od * od;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        e2 += __shfl_xor_sync(0xffffffffu, e2, off);
        r2 += __shfl_xor_sync(0xffffffffu, r2, off);
    }
    if (lane == 0) {
        red[0][warp] = e2;
        red[1][warp] = r2;
    }
    __syncthreads();
    if (tid == 0) {
        float a = 0.f, b = 0.f;
        for (int w = 0; w < kDgWarps; ++w) {
            a += red[0][w];
            b += red[1][w];
        }
        recall[orow] = Zst / Zt;
        err2[orow] = a;
        ref2[orow] = b;
    }
}

template <typename T, int D>
static int diag_impl(const void* Qp, const void* Kp, const void* Vp, svgear_dims qd, int Nk,
                     const int32_t* q_off, int Cq, const int32_t* k_off, int Ck,
                     const int32_t* pair_off, const int32_t* pair_kc, const void* O,
                     const int32_t* q_perm, float scale, const int32_t* rows, int R, float* recall,
                     float* err2, float* ref2, cudaStream_t st) {
    const int BH = qd.B * qd.H;
    diagnostics_kernel<T, D><<<dim3(R, BH), kDgThreads, Ck, st>>>(
        static_cast<const T*>(Qp), static_cast<const T*>(Kp), static_cast<const T*>(Vp), qd.N, Nk,
        q_off, Cq, k_off, Ck, pair_off, pair_kc, static_cast<const T*>(O), q_perm, scale, rows, R,
        recall, err2, ref2);
    count_launches(1);
    SVGEAR_LAUNCH_CHECK();
    return SVGEAR_OK;
}

int launch_diagnostics(const void* Qp, const void* Kp, const void* Vp, svgear_dims qd, int Nk,
                       const int32_t* q_off, int Cq, const int32_t* k_off, int Ck,
                       const int32_t* pair_off, const int32_t* pair_kc, const void* O,
                       const int32_t* q_perm, float scale, const int32_t* rows, int R,
                       float* recall, float* err2, float* ref2, cudaStream_t st) {
#define SVGEAR_DG(T, D)                                                                     \
    return diag_impl<T, D>(Qp, Kp, Vp, qd, Nk, q_off, Cq, k_off, Ck, pair_off, pair_kc, O,  \
                           q_perm, scale, rows, R, recall, err2, ref2, st)
    if (qd.dtype == SVGEAR_BF16) {
        if (qd.d == 128) SVGEAR_DG(__nv_bfloat16, 128);
        if (qd.d == 64) SVGEAR_DG(__nv_bfloat16, 64);
    } else if (qd.dtype == SVGEAR_F32) {
        if (qd.d == 128) SVGEAR_DG(float, 128);
        if (qd.d == 64) SVGEAR_DG(float, 64);
    }
#undef SVGEAR_DG
    return SVGEAR_ERR_UNSUPPORTED;
}

}  // namespace svgear
