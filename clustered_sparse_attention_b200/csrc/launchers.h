// launchers.h -- host-side launch functions of the library's kernels (internal).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "svgear.h"

namespace svgear {

// Tokens per block of the k-means++ D^2 pass and of the label sort.
constexpr int kKppTokens = 1024;
constexpr int kSortTokens = 1024;

inline int ceil_div(long long a, long long b) { return (int)((a + b - 1) / b); }

// api.cu: svgear_cluster on a range of heads of a larger call, drawing the
// k-means++ numbers of head bh from Philox stream sbase + bh.
int cluster_heads(const void* X, svgear_dims dims, int32_t C, int32_t iters,
                  const float* warm_centroids, uint64_t seed, uint64_t sbase, int32_t* labels,
                  int32_t* perm, int32_t* offsets, float* centroids, void* Xp, void* ws,
                  size_t ws_bytes, void* stream);

// guard.cu: the device's tensor-memory-lost word (address in the current
// context) and whether svgear_device_status has seen it set in this context.
int tmem_lost_word(int** out);
bool tmem_lost_latched();

// kmeans.cu
// k-means++ seeding: one cooperative persistent launch over a shared pool of
// work (see kpp_pool_kernel); err: device status words (4 ints).  Head bh of
// the launch draws from Philox stream sbase + bh (sbase = 0 for a whole call;
// a call on a range of heads passes the range's first flattened head).
int launch_kmeanspp(const void* X, svgear_dims dims, int C, uint64_t seed, uint64_t sbase,
                    float* centroids, int32_t* chosen, float* D2, int32_t* nearest, float* cc2,
                    double* blocksum, int32_t* counter /* 2 BH words */,
                    int32_t* gen /* BH + 1 words */, int* err,
                    cudaStream_t st);
// done[bh] != 0 skips head bh; changed[bh] is set to 1 when a label moves.
// scratch: assign_scratch_bytes(B*H, C, d, dtype) bytes (centroids re-laid
// for the kernel, and their norms).  bf16 tokens run on the tcgen05 kernel
// (assign_sm100.cu), whose bounded waits report through err (4 ints; f32
// tokens run on the SIMT kernel and never touch it).
int launch_assign(const void* X, svgear_dims dims, const float* centroids, int C,
                  int32_t* labels, void* scratch, int* err, cudaStream_t st,
                  const int32_t* done = nullptr, int32_t* changed = nullptr);
size_t assign_scratch_bytes(int BH, int C, int D, int dtype);
int launch_assign_sm100(const void* X, svgear_dims dims, const float* centroids, int C,
                        int32_t* labels, void* scratch, int* err, cudaStream_t st,
                        const int32_t* done, int32_t* changed);
size_t assign_sm100_scratch_bytes(int BH, int C, int D);
int launch_fixed_point(int32_t* changed, int32_t* done, int BH, cudaStream_t st);
// Recall and output error against dense attention on sampled query rows
// (diagnostics.cu).
int launch_diagnostics(const void* Qp, const void* Kp, const void* Vp, svgear_dims qd, int Nk,
                       const int32_t* q_off, int Cq, const int32_t* k_off, int Ck,
                       const int32_t* pair_off, const int32_t* pair_kc, const void* O,
                       const int32_t* q_perm, float scale, const int32_t* rows, int R,
                       float* recall, float* err2, float* ref2, cudaStream_t st);
// Per-coordinate population variance of every contiguous segment of X.
int launch_segment_var(const void* X, const int32_t* offsets, int C, svgear_dims dims,
                       float* out, cudaStream_t st);
// Mean of every segment; rows are perm[p] when perm != NULL (gather) else p.
// empty_zero: an empty segment writes zeros (else leaves the row untouched).
// scratch: segmean_scratch_bytes(B*H, N, d) bytes (partial sums of segments
// that cross position chunks).
int launch_segment_mean(const void* X, const int32_t* perm, const int32_t* offsets,
                        int C, svgear_dims dims, float* out, bool empty_zero, void* scratch,
                        cudaStream_t st, const int32_t* done = nullptr);
size_t segmean_scratch_bytes(int BH, int N, int D);
int launch_permute(const void* X, const int32_t* perm, svgear_dims dims, void* Xp,
                   cudaStream_t st);

// sort.cu
int launch_label_sort(const int32_t* labels, int BH, int N, int C, int32_t* perm,
                      int32_t* offsets, int32_t* block_hist, cudaStream_t st,
                      const int32_t* done = nullptr);

// route.cu
int launch_probe(const float* qbar, int Cq, const void* Kp, const void* Vp,
                 const float* kbar, const float* vbar, const int32_t* k_off, int Ck,
                 svgear_dims kdims, float scale, float* E, float* cmax, float* qT,
                 cudaStream_t st, bool value_free = false);
int launch_route_select(const float* E, const int32_t* q_off, int Cq, const int32_t* k_off,
                        int Ck, int BH, long long budget, const int32_t* budgets, int32_t* lists,
                        int32_t* counts, int32_t* pair_off, int32_t* pair_kc, cudaStream_t st);
// Top-p budget per query cluster (keys), budget int32 [BH][Cq].
int launch_topp_budget(const float* qbar, const int32_t* q_off, int Cq, const float* kbar,
                       const int32_t* k_off, int Ck, int BH, int D, double p, double scale,
                       int32_t* budget, cudaStream_t st);

// attend_sm100.cu: workspace of the tensor-core attention
struct AttendWs {
    int* status;                 // device status word (0 or SVGEAR_ERR_TIMEOUT)
    __nv_bfloat16* kbar16;       // [BH][Ck][d] bf16 key centroids
    __nv_bfloat16* vbar16;       // [BH][Ck][d] bf16 value centroids
    __nv_bfloat16* k2bar16;      // [BH][Ck][d] bf16 lambda*scale/2 * key variance
    int4* meta;                  // [BH][Cq] {segments, selected keys, skipped clusters, 0}
    int32_t* seg_prefix;         // [BH][Cq][Ck+1] list position of each segment
    int32_t* seg_row;            // [BH][Cq][Ck] first key row of each segment
    int32_t* comp_idx;           // [BH][Cq][Ck] skipped non-empty clusters
    float* comp_bias;            // [BH][Cq][Ck] log2(n_c) of those clusters
    int4* tiles;                 // [BH][maxT] {cluster, first row, end row, 0}: 128 or 256 rows
    int32_t* ntiles;             // [BH]
    int maxT;
};
int launch_attend_sm100(const void* Qp, const void* Kp, const void* Vp, svgear_dims qdims, int Nk,
                        const int32_t* q_off, int Cq, const int32_t* k_off, int Ck,
                        const int32_t* pair_off, const int32_t* pair_kc, const float* kbar,
                        const float* vbar, const int32_t* q_perm, float scale, void* O,
                        const float* kvar, float lambda, const AttendWs& w, cudaStream_t st);

// attend_simt.cu
// kvar (nullable): per-coordinate key variance [B*H][Ck][d]; a skipped
// cluster's score gains var_coef * sum_k q_k^2 kvar[c][k] (natural-log units).
int launch_attend_simt(const void* Qp, const void* Kp, const void* Vp, svgear_dims qdims,
                       int Nk, const int32_t* q_off, int Cq, const int32_t* k_off,
                       int Ck, const int32_t* pair_off, const int32_t* pair_kc,
                       const float* kbar, const float* vbar, const int32_t* q_perm,
                       float scale, void* O, const float* kvar, float var_coef, cudaStream_t st);

}  // namespace svgear
