// api.cu -- the C ABI declared in include/svgear.h: argument validation,
// workspace layout and the launch sequence of every entry point.
#include <math.h>
#include <string.h>

#include <atomic>

#include "carve.h"
#include "common.cuh"
#include "launchers.h"

using namespace svgear;

namespace svgear {
static std::atomic<unsigned long long> g_launches{0};
void count_launches(unsigned n) { g_launches.fetch_add(n, std::memory_order_relaxed); }
}  // namespace svgear

namespace {

inline size_t bh_of(const svgear_dims& d) { return (size_t)d.B * (size_t)d.H; }

int check_dims(const svgear_dims& d) {
    if (d.B < 0 || d.H < 0 || d.N < 1) return SVGEAR_ERR_INVALID_ARG;
    if (d.dtype != SVGEAR_F32 && d.dtype != SVGEAR_BF16) return SVGEAR_ERR_UNSUPPORTED;
    if (d.d != 64 && d.d != 128) return SVGEAR_ERR_UNSUPPORTED;
    if (bh_of(d) > 65535) return SVGEAR_ERR_UNSUPPORTED;   // grid y/z limit
    return SVGEAR_OK;
}

int check_C(int C, int N) {
    if (C < 1 || C > N) return SVGEAR_ERR_INVALID_ARG;
    if (C > SVGEAR_MAX_CLUSTERS) return SVGEAR_ERR_UNSUPPORTED;
    return SVGEAR_OK;
}

inline bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

struct KppWs {
    float* D2;
    double* blocksum;
    int32_t* chosen;
    int32_t* counter;
    int32_t* nearest;
    float* cc2;
    int32_t* gen;
};
KppWs carve_kpp(Carve& cv, const svgear_dims& d, int C) {
    KppWs w;
    w.D2 = cv.take<float>(bh_of(d) * d.N);
    w.blocksum = cv.take<double>(bh_of(d) * ceil_div(d.N, kKppTokens));
    w.chosen = cv.take<int32_t>(bh_of(d) * C);
    w.counter = cv.take<int32_t>(2 * bh_of(d));   // per-head 64-bit claim words
    w.nearest = cv.take<int32_t>(bh_of(d) * d.N);
    w.cc2 = cv.take<float>(bh_of(d) * C);
    w.gen = cv.take<int32_t>(bh_of(d) + 1);   // per-head arrivals, then the finished-head count
    return w;
}
int32_t* carve_sort(Carve& cv, const svgear_dims& d, int C) {
    return cv.take<int32_t>(bh_of(d) * ceil_div(d.N, kSortTokens) * (size_t)C);
}
void* carve_assign(Carve& cv, const svgear_dims& d, int C) {
    return cv.take<char>(assign_scratch_bytes((int)bh_of(d), C, d.d, d.dtype));
}
void* carve_segmean(Carve& cv, const svgear_dims& d) {
    return cv.take<char>(segmean_scratch_bytes((int)bh_of(d), d.N, d.d));
}
struct UpdWs {
    int32_t* perm;
    int32_t* offsets;
    int32_t* hist;
    void* segmean;
};
UpdWs carve_update(Carve& cv, const svgear_dims& d, int C) {
    UpdWs w;
    w.perm = cv.take<int32_t>(bh_of(d) * d.N);
    w.offsets = cv.take<int32_t>(bh_of(d) * (C + 1));
    w.hist = carve_sort(cv, d, C);
    w.segmean = carve_segmean(cv, d);
    return w;
}
struct SelWs {
    int32_t* lists;
    int32_t* counts;
};
SelWs carve_select(Carve& cv, size_t BH, int Cq, int Ck) {
    SelWs w;
    w.lists = cv.take<int32_t>(BH * Cq * (size_t)Ck);
    w.counts = cv.take<int32_t>(BH * Cq);
    return w;
}
struct RouteWs {
    float* E;
    float* cmax;   // the probe's maximum score per (probe, key cluster)
    float* qT;   // probes transposed in blocks of 128: [BH][ceil(Cq/128)][d][128]
    SelWs sel;
};
RouteWs carve_route(Carve& cv, size_t BH, int Cq, int Ck, int d) {
    RouteWs w;
    w.E = cv.take<float>(BH * Cq * (size_t)Ck);
    w.cmax = cv.take<float>(BH * Cq * (size_t)Ck);
    w.qT = cv.take<float>(BH * (size_t)ceil_div(Cq, 128) * 128 * (size_t)d);
    w.sel = carve_select(cv, BH, Cq, Ck);
    return w;
}

AttendWs carve_attend(Carve& cv, const svgear_dims& d, int Cq, int Ck) {
    AttendWs w;
    const size_t BH = bh_of(d);
    w.maxT = ceil_div(d.N, 128) + Cq;   // 128-row tiles per query cluster (enough for pairs)
    w.status = cv.take<int>(4);
    w.kbar16 = cv.take<__nv_bfloat16>(BH * Ck * (size_t)d.d);
    w.vbar16 = cv.take<__nv_bfloat16>(BH * Ck * (size_t)d.d);
    w.k2bar16 = cv.take<__nv_bfloat16>(BH * Ck * (size_t)d.d);
    w.meta = cv.take<int4>(BH * Cq);
    w.seg_prefix = cv.take<int32_t>(BH * Cq * (size_t)(Ck + 1));
    w.seg_row = cv.take<int32_t>(BH * Cq * (size_t)Ck);
    w.comp_idx = cv.take<int32_t>(BH * Cq * (size_t)Ck);
    w.comp_bias = cv.take<float>(BH * Cq * (size_t)Ck);
    w.tiles = cv.take<int4>(BH * (size_t)w.maxT);
    w.ntiles = cv.take<int32_t>(BH);
    return w;
}

// svgear_cluster's workspace: the device status words, per-head fixed-point
// flags, then the k-means++ scratch and the sort histograms and assignment
// scratch (used one after the other, so they overlap).
struct ClusterFlags {
    int* status;
    int32_t* done;
    int32_t* changed;
};
ClusterFlags carve_flags(Carve& cv, const svgear_dims& d) {
    ClusterFlags f;
    f.status = cv.take<int>(4);
    f.done = cv.take<int32_t>(bh_of(d));
    f.changed = cv.take<int32_t>(bh_of(d));
    return f;
}
size_t ws_cluster(const svgear_dims& d, int C) {
    Carve a(nullptr), b(nullptr);
    carve_flags(a, d);
    carve_flags(b, d);
    carve_kpp(a, d, C);
    carve_sort(b, d, C);
    carve_assign(b, d, C);
    carve_segmean(b, d);
    return (a.off > b.off ? a.off : b.off) + kAlign;
}

}  // namespace

extern "C" {

int32_t svgear_version(void) { return 100; }

uint64_t svgear_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

const char* svgear_status_string(int status) {
    switch (status) {
        case SVGEAR_OK: return "ok";
        case SVGEAR_ERR_INVALID_ARG: return "invalid argument";
        case SVGEAR_ERR_UNSUPPORTED: return "unsupported dtype, head dimension or size";
        case SVGEAR_ERR_CUDA: return "CUDA launch failed";
        case SVGEAR_ERR_TIMEOUT: return "device wait timed out";
        case SVGEAR_ERR_WORKSPACE: return "workspace too small";
        case SVGEAR_ERR_SCRATCH_LIMIT:
            return "sizes exceed the fixed scratch of the allocation-free entry point";
        case SVGEAR_ERR_TMEM_LOST:
            return "an earlier tensor-core kernel on this device kept its tensor memory after a "
                   "timeout; no tensor-core kernel can run in this context";
        default: return "unknown status";
    }
}

size_t svgear_workspace_bytes(int32_t op, svgear_dims dims, int32_t C1, int32_t C2) {
    if (check_dims(dims) != SVGEAR_OK) return 0;
    Carve cv(nullptr);
    switch (op) {
        case SVGEAR_OP_CLUSTER:
            if (check_C(C1, dims.N)) return 0;
            return ws_cluster(dims, C1);
        case SVGEAR_OP_KMEANSPP:
            if (check_C(C1, dims.N)) return 0;
            cv.take<int>(4);
            carve_kpp(cv, dims, C1);
            break;
        case SVGEAR_OP_LABEL_SORT:
            if (check_C(C1, dims.N)) return 0;
            carve_sort(cv, dims, C1);
            break;
        case SVGEAR_OP_KMEANS_UPDATE:
            if (check_C(C1, dims.N)) return 0;
            carve_update(cv, dims, C1);
            break;
        case SVGEAR_OP_KMEANS_ASSIGN:
            if (check_C(C1, dims.N)) return 0;
            cv.take<int>(4);
            carve_assign(cv, dims, C1);
            break;
        case SVGEAR_OP_CENTROIDS:
            if (check_C(C1, dims.N)) return 0;
            carve_segmean(cv, dims);
            break;
        case SVGEAR_OP_ROUTE:
            if (C1 < 1 || C2 < 1 || C1 > SVGEAR_MAX_CLUSTERS || C2 > SVGEAR_MAX_CLUSTERS) return 0;
            carve_route(cv, bh_of(dims), C1, C2, dims.d);
            break;
        case SVGEAR_OP_ROUTE_TOPP:
            if (C1 < 1 || C2 < 1 || C1 > SVGEAR_MAX_CLUSTERS || C2 > SVGEAR_MAX_CLUSTERS) return 0;
            carve_route(cv, bh_of(dims), C1, C2, dims.d);
            cv.take<int32_t>(bh_of(dims) * C1);
            break;
        case SVGEAR_OP_ATTEND:
            if (C1 < 1 || C2 < 1 || C1 > SVGEAR_MAX_CLUSTERS || C2 > SVGEAR_MAX_CLUSTERS) return 0;
            carve_attend(cv, dims, C1, C2);
            break;
        default:
            return 0;
    }
    return cv.off + kAlign;
}

int svgear_kmeanspp_init(const void* X, svgear_dims dims, int32_t C, uint64_t seed,
                         float* centroids, int32_t* seed_index, void* ws, size_t ws_bytes,
                         void* stream) {
    int s = check_dims(dims);
    if (s) return s;
    if ((s = check_C(C, dims.N))) return s;
    if (!X || !centroids || !ws || !aligned16(X)) return SVGEAR_ERR_INVALID_ARG;
    if (ws_bytes < svgear_workspace_bytes(SVGEAR_OP_KMEANSPP, dims, C, 0)) return SVGEAR_ERR_WORKSPACE;
    if (bh_of(dims) == 0) return SVGEAR_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    Carve cv(ws);
    int* status = cv.take<int>(4);
    if (cudaMemsetAsync(status, 0, 4 * sizeof(int), st) != cudaSuccess) return SVGEAR_ERR_CUDA;
    KppWs w = carve_kpp(cv, dims, C);
    return launch_kmeanspp(X, dims, C, seed, 0, centroids,
                           seed_index ? seed_index : w.chosen, w.D2,
                           w.nearest, w.cc2, w.blocksum, w.counter, w.gen, status, st);
}

int svgear_kmeans_assign(const void* X, svgear_dims dims, const float* centroids, int32_t C,
                         int32_t* labels, void* ws, size_t ws_bytes, void* stream) {
    int s = check_dims(dims);
    if (s) return s;
    if ((s = check_C(C, dims.N))) return s;
    if (!X || !centroids || !labels || !ws || !aligned16(X) || !aligned16(centroids))
        return SVGEAR_ERR_INVALID_ARG;
    if (ws_bytes < svgear_workspace_bytes(SVGEAR_OP_KMEANS_ASSIGN, dims, C, 0))
        return SVGEAR_ERR_WORKSPACE;
    if (bh_of(dims) == 0) return SVGEAR_OK;
    if (dims.dtype == SVGEAR_BF16 && tmem_lost_latched()) return SVGEAR_ERR_TMEM_LOST;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    Carve cv(ws);
    int* status = cv.take<int>(4);
    if (cudaMemsetAsync(status, 0, 4 * sizeof(int), st) != cudaSuccess) return SVGEAR_ERR_CUDA;
    return launch_assign(X, dims, centroids, C, labels, carve_assign(cv, dims, C), status, st);
}

int svgear_label_sort(const int32_t* labels, svgear_dims dims, int32_t C, int32_t* perm,
                      int32_t* offsets, void* ws, size_t ws_bytes, void* stream) {
    svgear_dims d2 = dims;
    d2.d = 64;
    d2.dtype = SVGEAR_F32;   // ignored by this op
    int s = check_dims(d2);
    if (s) return s;
    if ((s = check_C(C, dims.N))) return s;
    if (!labels || !perm || !offsets || !ws) return SVGEAR_ERR_INVALID_ARG;
    if (ws_bytes < svgear_workspace_bytes(SVGEAR_OP_LABEL_SORT, d2, C, 0)) return SVGEAR_ERR_WORKSPACE;
    if (bh_of(dims) == 0) return SVGEAR_OK;
    Carve cv(ws);
    int32_t* hist = carve_sort(cv, d2, C);
    return launch_label_sort(labels, (int)bh_of(dims), dims.N, C, perm, offsets, hist,
                             static_cast<cudaStream_t>(stream));
}

int svgear_kmeans_update(const void* X, svgear_dims dims, const int32_t* labels, int32_t C,
                         float* centroids, void* ws, size_t ws_bytes, void* stream) {
    int s = check_dims(dims);
    if (s) return s;
    if ((s = check_C(C, dims.N))) return s;
    if (!X || !labels || !centroids || !ws || !aligned16(X)) return SVGEAR_ERR_INVALID_ARG;
    if (ws_bytes < svgear_workspace_bytes(SVGEAR_OP_KMEANS_UPDATE, dims, C, 0))
        return SVGEAR_ERR_WORKSPACE;
    if (bh_of(dims) == 0) return SVGEAR_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    Carve cv(ws);
    UpdWs w = carve_update(cv, dims, C);
    if ((s = launch_label_sort(labels, (int)bh_of(dims), dims.N, C, w.perm, w.offsets, w.hist, st)))
        return s;
    return launch_segment_mean(X, w.perm, w.offsets, C, dims, centroids, false, w.segmean, st);
}

int svgear_cluster(const void* X, svgear_dims dims, int32_t C, int32_t iters,
                   const float* warm_centroids, uint64_t seed, int32_t* labels, int32_t* perm,
                   int32_t* offsets, float* centroids, void* Xp, void* ws, size_t ws_bytes,
                   void* stream) {
    return svgear::cluster_heads(X, dims, C, iters, warm_centroids, seed, 0, labels, perm,
                                 offsets, centroids, Xp, ws, ws_bytes, stream);
}

}  // extern "C"

// svgear_cluster on a range of heads of a larger call: head bh of these dims
// draws its k-means++ numbers from Philox stream sbase + bh, so clustering
// the heads [h0, h1) with sbase = h0 repeats what a call on all heads gives
// them (every head's k-means is independent of the others').
int svgear::cluster_heads(const void* X, svgear_dims dims, int32_t C, int32_t iters,
                          const float* warm_centroids, uint64_t seed, uint64_t sbase,
                          int32_t* labels, int32_t* perm, int32_t* offsets, float* centroids,
                          void* Xp, void* ws, size_t ws_bytes, void* stream) {
    int s = check_dims(dims);
    if (s) return s;
    if ((s = check_C(C, dims.N))) return s;
    if (iters < 1) return SVGEAR_ERR_INVALID_ARG;
    if (!X || !labels || !perm || !offsets || !centroids || !ws || !aligned16(X) ||
        !aligned16(centroids) || (Xp && !aligned16(Xp)))
        return SVGEAR_ERR_INVALID_ARG;
    if (ws_bytes < svgear_workspace_bytes(SVGEAR_OP_CLUSTER, dims, C, 0)) return SVGEAR_ERR_WORKSPACE;
    if (bh_of(dims) == 0) return SVGEAR_OK;
    if (dims.dtype == SVGEAR_BF16 && tmem_lost_latched()) return SVGEAR_ERR_TMEM_LOST;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int BH = (int)bh_of(dims);
    Carve cf(ws);
    ClusterFlags fl = carve_flags(cf, dims);
    const size_t flag_bytes = (size_t)((char*)fl.changed - (char*)fl.status) + sizeof(int32_t) * BH;
    if (cudaMemsetAsync(fl.status, 0, flag_bytes, st) != cudaSuccess) return SVGEAR_ERR_CUDA;
    if (warm_centroids) {
        if (warm_centroids != centroids &&
            cudaMemcpyAsync(centroids, warm_centroids, sizeof(float) * BH * (size_t)C * dims.d,
                            cudaMemcpyDeviceToDevice, st) != cudaSuccess)
            return SVGEAR_ERR_CUDA;
    } else {
        Carve cv(ws);
        carve_flags(cv, dims);
        KppWs w = carve_kpp(cv, dims, C);
        if ((s = launch_kmeanspp(X, dims, C, seed, sbase, centroids, w.chosen, w.D2,
                                 w.nearest,
                                 w.cc2,
                                 w.blocksum, w.counter, w.gen, fl.status, st)))
            return s;
    }
    Carve cv(ws);
    carve_flags(cv, dims);
    int32_t* hist = carve_sort(cv, dims, C);
    void* ascratch = carve_assign(cv, dims, C);
    void* mscratch = carve_segmean(cv, dims);
    // Lloyd rounds.  From the second round on, a head whose assignment moved
    // no label has reached the fixed point (the sort and the deterministic
    // update would reproduce the current perm, offsets and centroids), so its
    // remaining kernels return at once; the results are those of all rounds.
    for (int it = 0; it < iters; ++it) {
        const bool track = it > 0;
        if ((s = launch_assign(X, dims, centroids, C, labels, ascratch, fl.status, st, fl.done,
                               track ? fl.changed : nullptr)))
            return s;
        if (track && (s = launch_fixed_point(fl.changed, fl.done, BH, st))) return s;
        if ((s = launch_label_sort(labels, BH, dims.N, C, perm, offsets, hist, st, fl.done)))
            return s;
        if ((s = launch_segment_mean(X, perm, offsets, C, dims, centroids, false, mscratch, st,
                                     fl.done)))
            return s;
    }
    if (Xp) return launch_permute(X, perm, dims, Xp, st);
    return SVGEAR_OK;
}

extern "C" {

int svgear_permute(const void* X, const int32_t* perm, svgear_dims dims, void* Xp, void* stream) {
    int s = check_dims(dims);
    if (s) return s;
    if (!X || !perm || !Xp || !aligned16(X) || !aligned16(Xp)) return SVGEAR_ERR_INVALID_ARG;
    if (bh_of(dims) == 0) return SVGEAR_OK;
    return launch_permute(X, perm, dims, Xp, static_cast<cudaStream_t>(stream));
}

int svgear_centroids(const void* Xp, const int32_t* offsets, int32_t C, svgear_dims dims,
                     float* centroids, void* ws, size_t ws_bytes, void* stream) {
    int s = check_dims(dims);
    if (s) return s;
    if ((s = check_C(C, dims.N))) return s;
    if (!Xp || !offsets || !centroids || !ws || !aligned16(Xp)) return SVGEAR_ERR_INVALID_ARG;
    if (ws_bytes < svgear_workspace_bytes(SVGEAR_OP_CENTROIDS, dims, C, 0))
        return SVGEAR_ERR_WORKSPACE;
    if (bh_of(dims) == 0) return SVGEAR_OK;
    Carve cv(ws);
    return launch_segment_mean(Xp, nullptr, offsets, C, dims, centroids, true,
                               carve_segmean(cv, dims), static_cast<cudaStream_t>(stream));
}

static int check_route_common(int Cq, int Ck, int Nk, float density) {
    if (Cq < 1 || Ck < 1 || Ck > Nk) return SVGEAR_ERR_INVALID_ARG;
    if (Cq > SVGEAR_MAX_CLUSTERS || Ck > SVGEAR_MAX_CLUSTERS) return SVGEAR_ERR_UNSUPPORTED;
    if (!(density > 0.f && density <= 1.f)) return SVGEAR_ERR_INVALID_ARG;
    return SVGEAR_OK;
}

int svgear_probe(const float* qbar, int32_t Cq, const void* Kp, const void* Vp, const float* kbar,
                 const float* vbar, const int32_t* k_off, int32_t Ck, svgear_dims kdims,
                 float scale, float* E, void* ws, size_t ws_bytes, void* stream) {
    int s = check_dims(kdims);
    if (s) return s;
    if ((s = check_route_common(Cq, Ck, kdims.N, 1.f))) return s;
    if (!qbar || !Kp || !Vp || !kbar || !vbar || !k_off || !E || !ws || !aligned16(Kp) ||
        !aligned16(Vp) || !isfinite(scale))
        return SVGEAR_ERR_INVALID_ARG;
    if (ws_bytes < svgear_workspace_bytes(SVGEAR_OP_ROUTE, kdims, Cq, Ck)) return SVGEAR_ERR_WORKSPACE;
    if (bh_of(kdims) == 0) return SVGEAR_OK;
    Carve cv(ws);
    RouteWs w = carve_route(cv, bh_of(kdims), Cq, Ck, kdims.d);
    return launch_probe(qbar, Cq, Kp, Vp, kbar, vbar, k_off, Ck, kdims, scale, E, w.cmax, w.qT,
                        static_cast<cudaStream_t>(stream));
}

int svgear_route_select(const float* E, const int32_t* q_off, int32_t Cq, const int32_t* k_off,
                        int32_t Ck, int32_t B, int32_t H, int32_t Nk, float density,
                        int32_t* pair_off, int32_t* pair_kc, void* ws, size_t ws_bytes,
                        void* stream) {
    if (B < 0 || H < 0 || Nk < 1) return SVGEAR_ERR_INVALID_ARG;
    const size_t BH = (size_t)B * H;
    if (BH > 65535) return SVGEAR_ERR_UNSUPPORTED;
    int s = check_route_common(Cq, Ck, Nk, density);
    if (s) return s;
    if (!E || !q_off || !k_off || !pair_off || !pair_kc || !ws) return SVGEAR_ERR_INVALID_ARG;
    Carve need(nullptr);
    carve_select(need, BH, Cq, Ck);
    if (ws_bytes < need.off + kAlign) return SVGEAR_ERR_WORKSPACE;
    if (BH == 0) return SVGEAR_OK;
    Carve cv(ws);
    SelWs w = carve_select(cv, BH, Cq, Ck);
    const long long budget = (long long)floor((double)density * (double)Nk);
    return launch_route_select(E, q_off, Cq, k_off, Ck, (int)BH, budget, nullptr, w.lists,
                               w.counts, pair_off, pair_kc, static_cast<cudaStream_t>(stream));
}

int svgear_route(const float* qbar, const int32_t* q_off, int32_t Cq, const float* kbar,
                 const float* vbar, const int32_t* k_off, int32_t Ck, const void* Kp,
                 const void* Vp, svgear_dims kdims, float density, float scale,
                 int32_t* pair_off, int32_t* pair_kc, float* E_out, void* ws, size_t ws_bytes,
                 void* stream) {
    int s = check_dims(kdims);
    if (s) return s;
    if ((s = check_route_common(Cq, Ck, kdims.N, density))) return s;
    if (!qbar || !q_off || !kbar || !vbar || !k_off || !Kp || !Vp || !pair_off || !pair_kc ||
        !ws || !aligned16(Kp) || !aligned16(Vp) || !isfinite(scale))
        return SVGEAR_ERR_INVALID_ARG;
    if (ws_bytes < svgear_workspace_bytes(SVGEAR_OP_ROUTE, kdims, Cq, Ck)) return SVGEAR_ERR_WORKSPACE;
    if (bh_of(kdims) == 0) return SVGEAR_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    Carve cv(ws);
    RouteWs w = carve_route(cv, bh_of(kdims), Cq, Ck, kdims.d);
    float* E = E_out ? E_out : w.E;
    if ((s = launch_probe(qbar, Cq, Kp, Vp, kbar, vbar, k_off, Ck, kdims, scale, E, w.cmax, w.qT, st)))
        return s;
    const long long budget = (long long)floor((double)density * (double)kdims.N);
    return launch_route_select(E, q_off, Cq, k_off, Ck, (int)bh_of(kdims), budget, nullptr,
                               w.sel.lists, w.sel.counts, pair_off, pair_kc, st);
}

int svgear_topp_budget(const float* qbar, const int32_t* q_off, int32_t Cq, const float* kbar,
                       const int32_t* k_off, int32_t Ck, int32_t B, int32_t H, int32_t d,
                       int32_t Nk, float p, float scale, int32_t* budget, void* stream) {
    if (B < 0 || H < 0 || Nk < 1) return SVGEAR_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return SVGEAR_ERR_UNSUPPORTED;
    const size_t BH = (size_t)B * H;
    if (BH > 65535) return SVGEAR_ERR_UNSUPPORTED;
    int s = check_route_common(Cq, Ck, Nk, p);
    if (s) return s;
    if (!qbar || !q_off || !kbar || !k_off || !budget || !isfinite(scale)) return SVGEAR_ERR_INVALID_ARG;
    if (BH == 0) return SVGEAR_OK;
    return launch_topp_budget(qbar, q_off, Cq, kbar, k_off, Ck, (int)BH, d, (double)p,
                              (double)scale, budget, static_cast<cudaStream_t>(stream));
}

int svgear_route_select_budget(const float* E, const int32_t* q_off, int32_t Cq,
                               const int32_t* k_off, int32_t Ck, int32_t B, int32_t H,
                               int32_t Nk, const int32_t* budget, int32_t* pair_off,
                               int32_t* pair_kc, void* ws, size_t ws_bytes, void* stream) {
    if (B < 0 || H < 0 || Nk < 1) return SVGEAR_ERR_INVALID_ARG;
    const size_t BH = (size_t)B * H;
    if (BH > 65535) return SVGEAR_ERR_UNSUPPORTED;
    int s = check_route_common(Cq, Ck, Nk, 1.f);
    if (s) return s;
    if (!E || !q_off || !k_off || !budget || !pair_off || !pair_kc || !ws)
        return SVGEAR_ERR_INVALID_ARG;
    Carve need(nullptr);
    carve_select(need, BH, Cq, Ck);
    if (ws_bytes < need.off + kAlign) return SVGEAR_ERR_WORKSPACE;
    if (BH == 0) return SVGEAR_OK;
    Carve cv(ws);
    SelWs w = carve_select(cv, BH, Cq, Ck);
    return launch_route_select(E, q_off, Cq, k_off, Ck, (int)BH, 0, budget, w.lists, w.counts,
                               pair_off, pair_kc, static_cast<cudaStream_t>(stream));
}

int svgear_route_topp(const float* qbar, const int32_t* q_off, int32_t Cq, const float* kbar,
                      const float* vbar, const int32_t* k_off, int32_t Ck, const void* Kp,
                      const void* Vp, svgear_dims kdims, float p, float scale, int32_t* pair_off,
                      int32_t* pair_kc, float* E_out, int32_t* budget_out, void* ws,
                      size_t ws_bytes, void* stream) {
    int s = check_dims(kdims);
    if (s) return s;
    if ((s = check_route_common(Cq, Ck, kdims.N, p))) return s;
    if (!qbar || !q_off || !kbar || !vbar || !k_off || !Kp || !Vp || !pair_off || !pair_kc ||
        !ws || !aligned16(Kp) || !aligned16(Vp) || !isfinite(scale))
        return SVGEAR_ERR_INVALID_ARG;
    if (ws_bytes < svgear_workspace_bytes(SVGEAR_OP_ROUTE_TOPP, kdims, Cq, Ck))
        return SVGEAR_ERR_WORKSPACE;
    if (bh_of(kdims) == 0) return SVGEAR_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    Carve cv(ws);
    RouteWs w = carve_route(cv, bh_of(kdims), Cq, Ck, kdims.d);
    int32_t* bud = cv.take<int32_t>(bh_of(kdims) * Cq);
    if (budget_out) bud = budget_out;
    float* E = E_out ? E_out : w.E;
    if ((s = launch_probe(qbar, Cq, Kp, Vp, kbar, vbar, k_off, Ck, kdims, scale, E, w.cmax, w.qT, st)))
        return s;
    if ((s = launch_topp_budget(qbar, q_off, Cq, kbar, k_off, Ck, (int)bh_of(kdims), kdims.d,
                                (double)p, (double)scale, bud, st)))
        return s;
    return launch_route_select(E, q_off, Cq, k_off, Ck, (int)bh_of(kdims), 0, bud, w.sel.lists,
                               w.sel.counts, pair_off, pair_kc, st);
}

int svgear_attend_var(const void* Qp, const void* Kp, const void* Vp, svgear_dims qdims,
                      int32_t Nk, const int32_t* q_off, int32_t Cq, const int32_t* k_off,
                      int32_t Ck, const int32_t* pair_off, const int32_t* pair_kc,
                      const float* kbar, const float* vbar, const float* kvar, float lambda,
                      const int32_t* q_perm, float scale, void* O, void* ws, size_t ws_bytes,
                      void* stream) {
    int s = check_dims(qdims);
    if (s) return s;
    if (Nk < 1) return SVGEAR_ERR_INVALID_ARG;
    if ((s = check_route_common(Cq, Ck, Nk, 1.f))) return s;
    if (Cq > qdims.N) return SVGEAR_ERR_INVALID_ARG;
    if (!Qp || !Kp || !Vp || !q_off || !k_off || !pair_off || !pair_kc || !kbar || !vbar ||
        !q_perm || !O || !ws || !aligned16(Qp) || !aligned16(Kp) || !aligned16(Vp) ||
        !aligned16(O) || !isfinite(scale) || !isfinite(lambda))
        return SVGEAR_ERR_INVALID_ARG;
    if (ws_bytes < svgear_workspace_bytes(SVGEAR_OP_ATTEND, qdims, Cq, Ck)) return SVGEAR_ERR_WORKSPACE;
    if (bh_of(qdims) == 0) return SVGEAR_OK;
    if (qdims.dtype == SVGEAR_BF16 && tmem_lost_latched()) return SVGEAR_ERR_TMEM_LOST;
    if (lambda == 0.f) kvar = nullptr;   // plain SVG-EAR compensation
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    Carve cv(ws);
    AttendWs w = carve_attend(cv, qdims, Cq, Ck);
    if (qdims.dtype == SVGEAR_BF16)
        return launch_attend_sm100(Qp, Kp, Vp, qdims, Nk, q_off, Cq, k_off, Ck, pair_off, pair_kc,
                                   kbar, vbar, q_perm, scale, O, kvar, lambda, w, st);
    if (cudaMemsetAsync(w.status, 0, 4 * sizeof(int), st) != cudaSuccess) return SVGEAR_ERR_CUDA;
    return launch_attend_simt(Qp, Kp, Vp, qdims, Nk, q_off, Cq, k_off, Ck, pair_off, pair_kc, kbar,
                              vbar, q_perm, scale, O, kvar, lambda * scale * scale * 0.5f, st);
}

int svgear_attend(const void* Qp, const void* Kp, const void* Vp, svgear_dims qdims, int32_t Nk,
                  const int32_t* q_off, int32_t Cq, const int32_t* k_off, int32_t Ck,
                  const int32_t* pair_off, const int32_t* pair_kc, const float* kbar,
                  const float* vbar, const int32_t* q_perm, float scale, void* O, void* ws,
                  size_t ws_bytes, void* stream) {
    return svgear_attend_var(Qp, Kp, Vp, qdims, Nk, q_off, Cq, k_off, Ck, pair_off, pair_kc, kbar,
                             vbar, nullptr, 0.f, q_perm, scale, O, ws, ws_bytes, stream);
}

int svgear_probe_value_free(const float* qbar, int32_t Cq, const void* Kp, const float* kbar,
                            const int32_t* k_off, int32_t Ck, svgear_dims kdims, float scale,
                            float* E, void* ws, size_t ws_bytes, void* stream) {
    int s = check_dims(kdims);
    if (s) return s;
    if ((s = check_route_common(Cq, Ck, kdims.N, 1.f))) return s;
    if (!qbar || !Kp || !kbar || !k_off || !E || !ws || !aligned16(Kp) || !isfinite(scale))
        return SVGEAR_ERR_INVALID_ARG;
    if (ws_bytes < svgear_workspace_bytes(SVGEAR_OP_ROUTE, kdims, Cq, Ck)) return SVGEAR_ERR_WORKSPACE;
    if (bh_of(kdims) == 0) return SVGEAR_OK;
    Carve cv(ws);
    RouteWs w = carve_route(cv, bh_of(kdims), Cq, Ck, kdims.d);
    return launch_probe(qbar, Cq, Kp, nullptr, kbar, nullptr, k_off, Ck, kdims, scale, E,
                        w.cmax, w.qT, static_cast<cudaStream_t>(stream), true);
}

int svgear_diagnostics(const void* Qp, const void* Kp, const void* Vp, svgear_dims qdims,
                       int32_t Nk, const int32_t* q_off, int32_t Cq, const int32_t* k_off,
                       int32_t Ck, const int32_t* pair_off, const int32_t* pair_kc, const void* O,
                       const int32_t* q_perm, float scale, const int32_t* rows, int32_t R,
                       float* recall, float* err2, float* ref2, void* stream) {
    int s = check_dims(qdims);
    if (s) return s;
    if (Nk < 1 || R < 0) return SVGEAR_ERR_INVALID_ARG;
    if ((s = check_route_common(Cq, Ck, Nk, 1.f))) return s;
    if (!Qp || !Kp || !Vp || !q_off || !k_off || !pair_off || !pair_kc || !O || !q_perm ||
        !rows || !recall || !err2 || !ref2 || !isfinite(scale))
        return SVGEAR_ERR_INVALID_ARG;
    if (bh_of(qdims) == 0 || R == 0) return SVGEAR_OK;
    return launch_diagnostics(Qp, Kp, Vp, qdims, Nk, q_off, Cq, k_off, Ck, pair_off, pair_kc, O,
                              q_perm, scale, rows, R, recall, err2, ref2,
                              static_cast<cudaStream_t>(stream));
}

int svgear_key_variance(const void* Kp, const int32_t* k_off, int32_t Ck, svgear_dims kdims,
                        float* kvar, void* stream) {
    int s = check_dims(kdims);
    if (s) return s;
    if ((s = check_C(Ck, kdims.N))) return s;
    if (!Kp || !k_off || !kvar || !aligned16(Kp)) return SVGEAR_ERR_INVALID_ARG;
    if (bh_of(kdims) == 0) return SVGEAR_OK;
    return launch_segment_var(Kp, k_off, Ck, kdims, kvar, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
