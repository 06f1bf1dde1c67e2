// layer.cu -- one whole layer call behind the C ABI: svgear_layer on device
// buffers and svgear_layer_host on host buffers (the copies inside the call).
//
// The layer composes the public entry points in the order the method runs
// them ([TASK] the three routines and the agent's steps 1-3; [SVG2] section
// 3.4): k-means on Q and on K with the permutation, the permuted values and
// their cluster means, the probe with greedy routing, and the attention pass
// with centroid compensation, O back in the original token order.  Every
// buffer it needs is carved from the caller's workspace; the host variant
// adds the device copies of Q, K and V (O reuses Q's copy, which nothing
// reads once Q is clustered).
#include <math.h>

#include "carve.h"
#include "common.cuh"
#include "launchers.h"

using namespace svgear;

namespace {

inline size_t bh_of(const svgear_dims& d) { return (size_t)d.B * (size_t)d.H; }

size_t tensor_bytes(const svgear_dims& d) {
    return bh_of(d) * (size_t)d.N * (size_t)d.d * (d.dtype == SVGEAR_BF16 ? 2 : 4);
}

int check_params(const svgear_dims& d, const svgear_layer_params* p) {
    if (!p) return SVGEAR_ERR_INVALID_ARG;
    if (d.B < 0 || d.H < 0 || d.N < 1) return SVGEAR_ERR_INVALID_ARG;
    if (d.dtype != SVGEAR_F32 && d.dtype != SVGEAR_BF16) return SVGEAR_ERR_UNSUPPORTED;
    if (d.d != 64 && d.d != 128) return SVGEAR_ERR_UNSUPPORTED;
    if (bh_of(d) > 65535) return SVGEAR_ERR_UNSUPPORTED;
    if (p->Cq < 1 || p->Ck < 1 || p->Cq > d.N || p->Ck > d.N) return SVGEAR_ERR_INVALID_ARG;
    if (p->Cq > SVGEAR_MAX_CLUSTERS || p->Ck > SVGEAR_MAX_CLUSTERS) return SVGEAR_ERR_UNSUPPORTED;
    if (p->iters < 1) return SVGEAR_ERR_INVALID_ARG;
    if (!(p->topp >= 0.f && p->topp <= 1.f)) return SVGEAR_ERR_INVALID_ARG;
    if (p->topp == 0.f && !(p->density > 0.f && p->density <= 1.f)) return SVGEAR_ERR_INVALID_ARG;
    if (!isfinite(p->scale) || !isfinite(p->var_lambda)) return SVGEAR_ERR_INVALID_ARG;
    return SVGEAR_OK;
}

// Everything one call keeps alive, then one scratch region that the stages
// use one after the other (cluster Q, cluster K, route, attend).
struct LayerWs {
    void* Qd;   // host variant: device copies of the inputs (O reuses Qd)
    void* Kd;
    void* Vd;
    int32_t *labels_q, *perm_q, *off_q, *labels_k, *perm_k, *off_k;
    float *cent_q, *cent_k, *vbar, *kvar;
    void *Xp_q, *Xp_k, *Vp;
    int32_t *pair_off, *pair_kc;
    void* scratch;
    size_t scratch_bytes;
};

size_t scratch_need(const svgear_dims& d, const svgear_layer_params* p) {
    size_t s = svgear_workspace_bytes(SVGEAR_OP_CLUSTER, d, p->Cq, 0);
    size_t t = svgear_workspace_bytes(SVGEAR_OP_CLUSTER, d, p->Ck, 0);
    if (t > s) s = t;
    t = svgear_workspace_bytes(p->topp > 0.f ? SVGEAR_OP_ROUTE_TOPP : SVGEAR_OP_ROUTE, d, p->Cq,
                               p->Ck);
    if (t > s) s = t;
    t = svgear_workspace_bytes(SVGEAR_OP_ATTEND, d, p->Cq, p->Ck);
    if (t > s) s = t;
    t = svgear_workspace_bytes(SVGEAR_OP_CENTROIDS, d, p->Ck, 0);
    if (t > s) s = t;
    return s;
}

LayerWs carve_layer(Carve& cv, const svgear_dims& d, const svgear_layer_params* p, bool host) {
    LayerWs w = {};
    const size_t BH = bh_of(d), N = (size_t)d.N, D = (size_t)d.d;
    const size_t tb = tensor_bytes(d);
    if (host) {
        w.Qd = cv.take<char>(tb);
        w.Kd = cv.take<char>(tb);
        w.Vd = cv.take<char>(tb);
    }
    w.labels_q = cv.take<int32_t>(BH * N);
    w.perm_q = cv.take<int32_t>(BH * N);
    w.off_q = cv.take<int32_t>(BH * (p->Cq + 1));
    w.cent_q = cv.take<float>(BH * p->Cq * D);
    w.Xp_q = cv.take<char>(tb);
    w.labels_k = cv.take<int32_t>(BH * N);
    w.perm_k = cv.take<int32_t>(BH * N);
    w.off_k = cv.take<int32_t>(BH * (p->Ck + 1));
    w.cent_k = cv.take<float>(BH * p->Ck * D);
    w.Xp_k = cv.take<char>(tb);
    w.Vp = cv.take<char>(tb);
    w.vbar = cv.take<float>(BH * p->Ck * D);
    w.kvar = p->var_lambda != 0.f ? cv.take<float>(BH * p->Ck * D) : nullptr;
    w.pair_off = cv.take<int32_t>(BH * (p->Cq + 1));
    w.pair_kc = cv.take<int32_t>(BH * p->Cq * (size_t)p->Ck);
    w.scratch_bytes = scratch_need(d, p);
    w.scratch = cv.take<char>(w.scratch_bytes);
    return w;
}

inline int record(void* const* ev, int i, cudaStream_t st) {
    if (!ev || !ev[i]) return SVGEAR_OK;
    return cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), st) == cudaSuccess ? SVGEAR_OK
                                                                              : SVGEAR_ERR_CUDA;
}

inline int wait_on(cudaEvent_t ev, cudaStream_t st) {
    if (!ev) return SVGEAR_OK;
    return cudaStreamWaitEvent(st, ev, 0) == cudaSuccess ? SVGEAR_OK : SVGEAR_ERR_CUDA;
}

// The stages on `st`.  ready[0..2] (nullable): events the stream waits for
// before the first read of Q, K and V (inputs still arriving on another
// stream).  cq_out / ck_out: the caller's centroid outputs, or NULL.
int run_layer(const void* Q, const void* K, const void* V, svgear_dims dims,
              const svgear_layer_params* p, const float* warm_q, const float* warm_k, void* O,
              float* cq_out, float* ck_out, const LayerWs& w, void* const* ev,
              const cudaEvent_t* ready, cudaStream_t st) {
    int s;
    void* vst = static_cast<void*>(st);
    float* cent_q = cq_out ? cq_out : w.cent_q;
    float* cent_k = ck_out ? ck_out : w.cent_k;
    if ((s = record(ev, 0, st))) return s;
    if (ready && (s = wait_on(ready[0], st))) return s;
    if ((s = svgear_cluster(Q, dims, p->Cq, p->iters, warm_q, 2 * p->seed, w.labels_q, w.perm_q,
                            w.off_q, cent_q, w.Xp_q, w.scratch, w.scratch_bytes, vst)))
        return s;
    if ((s = record(ev, 1, st))) return s;
    if (ready && (s = wait_on(ready[1], st))) return s;
    if ((s = svgear_cluster(K, dims, p->Ck, p->iters, warm_k, 2 * p->seed + 1, w.labels_k,
                            w.perm_k, w.off_k, cent_k, w.Xp_k, w.scratch, w.scratch_bytes, vst)))
        return s;
    if ((s = record(ev, 2, st))) return s;
    if (ready && (s = wait_on(ready[2], st))) return s;
    if ((s = svgear_permute(V, w.perm_k, dims, w.Vp, vst))) return s;
    if ((s = svgear_centroids(w.Vp, w.off_k, p->Ck, dims, w.vbar, w.scratch, w.scratch_bytes,
                              vst)))
        return s;
    if ((s = record(ev, 3, st))) return s;
    if (p->topp > 0.f)
        s = svgear_route_topp(cent_q, w.off_q, p->Cq, cent_k, w.vbar, w.off_k, p->Ck, w.Xp_k, w.Vp,
                              dims, p->topp, p->scale, w.pair_off, w.pair_kc, nullptr, nullptr,
                              w.scratch, w.scratch_bytes, vst);
    else
        s = svgear_route(cent_q, w.off_q, p->Cq, cent_k, w.vbar, w.off_k, p->Ck, w.Xp_k, w.Vp, dims,
                         p->density, p->scale, w.pair_off, w.pair_kc, nullptr, w.scratch,
                         w.scratch_bytes, vst);
    if (s) return s;
    if ((s = record(ev, 4, st))) return s;
    if (w.kvar && (s = svgear_key_variance(w.Xp_k, w.off_k, p->Ck, dims, w.kvar, vst))) return s;
    if ((s = svgear_attend_var(w.Xp_q, w.Xp_k, w.Vp, dims, dims.N, w.off_q, p->Cq, w.off_k, p->Ck,
                               w.pair_off, w.pair_kc, cent_k, w.vbar, w.kvar, p->var_lambda,
                               w.perm_q, p->scale, O, w.scratch, w.scratch_bytes, vst)))
        return s;
    return record(ev, 5, st);
}

// The host-buffer layer as a pipeline over head groups (flattened b*H + h):
// the inputs go up on a copy stream, Q in kQGroups parts, then K and V; Q is
// clustered part by part as it arrives (each part's k-means++ draws from the
// Philox streams of its own heads, so the result is the whole call's), K, V,
// the value centroids and routing run whole, and attention runs in kOGroups
// parts whose O goes back to the host on a third stream while the next part
// is computed.  So only the first part of Q and the last part of O cross the
// host link with nothing to overlap.  The copy stream first waits for all
// work already on `st` (an earlier call may still read this workspace); the
// call's streams and events are released once their work is done.
struct HostPipeline {
    // Q parts: each clusters at least 8 heads (k-means++ of fewer heads is
    // bound by its per-seed latency); O parts: the smaller the last one, the
    // less of O crosses the host link with nothing to overlap
    static constexpr int kQGroups = 2, kOGroups = 8;
    static constexpr int kMinHeadsQ = 8, kMinHeadsO = 4;
    cudaStream_t xs = nullptr, ds = nullptr;
    cudaEvent_t entry = nullptr, done_d2h = nullptr, k_ready = nullptr, v_ready = nullptr;
    cudaEvent_t q_ready[kQGroups] = {}, o_ready[kOGroups] = {};

    static int groups(int BH, int want, int min_heads) {
        int g = BH / min_heads;
        return g < 1 ? 1 : (g > want ? want : g);
    }
    // heads [lo, hi) of group g of G over BH (contiguous, sizes within one)
    static void range(int BH, int G, int g, int* lo, int* hi) {
        const int base = BH / G, extra = BH % G;
        *lo = g * base + (g < extra ? g : extra);
        *hi = *lo + base + (g < extra ? 1 : 0);
    }
    bool create() {
        auto ev = [](cudaEvent_t* e) {
            return cudaEventCreateWithFlags(e, cudaEventDisableTiming) == cudaSuccess;
        };
        bool ok = cudaStreamCreateWithFlags(&xs, cudaStreamNonBlocking) == cudaSuccess &&
                  cudaStreamCreateWithFlags(&ds, cudaStreamNonBlocking) == cudaSuccess &&
                  ev(&entry) && ev(&done_d2h) && ev(&k_ready) && ev(&v_ready);
        for (cudaEvent_t& e : q_ready) ok = ok && ev(&e);
        for (cudaEvent_t& e : o_ready) ok = ok && ev(&e);
        return ok;
    }
    void release() {
        cudaEvent_t all[] = {entry, done_d2h, k_ready, v_ready};
        for (cudaEvent_t e : all)
            if (e) cudaEventDestroy(e);
        for (cudaEvent_t e : q_ready)
            if (e) cudaEventDestroy(e);
        for (cudaEvent_t e : o_ready)
            if (e) cudaEventDestroy(e);
        if (xs) cudaStreamDestroy(xs);
        if (ds) cudaStreamDestroy(ds);
    }

    int run(const void* Qh, const void* Kh, const void* Vh, svgear_dims dims,
            const svgear_layer_params* p, const float* warm_q, const float* warm_k, void* Oh,
            float* cq_out, float* ck_out, const LayerWs& w, cudaStream_t st) {
        if (!create()) return SVGEAR_ERR_CUDA;
        int s;
        void* vst = static_cast<void*>(st);
        const int BH = (int)bh_of(dims), N = dims.N, D = dims.d;
        const size_t esz = dims.dtype == SVGEAR_BF16 ? 2 : 4;
        const size_t head_bytes = (size_t)N * D * esz, tb = tensor_bytes(dims);
        float* cent_q = cq_out ? cq_out : w.cent_q;
        float* cent_k = ck_out ? ck_out : w.cent_k;
        const int GQ = groups(BH, kQGroups, kMinHeadsQ), GO = groups(BH, kOGroups, kMinHeadsO);
        auto sub = [&](int lo, int hi) {   // dims of the flattened heads [lo, hi)
            svgear_dims d = dims;
            d.B = 1;
            d.H = hi - lo;
            return d;
        };
        auto at = [](const void* base, size_t off) {
            return static_cast<void*>(static_cast<char*>(const_cast<void*>(base)) + off);
        };
        // inputs
        if (cudaEventRecord(entry, st) != cudaSuccess || cudaStreamWaitEvent(xs, entry, 0) != cudaSuccess)
            return SVGEAR_ERR_CUDA;
        for (int g = 0; g < GQ; ++g) {
            int lo, hi;
            range(BH, GQ, g, &lo, &hi);
            if (cudaMemcpyAsync(at(w.Qd, lo * head_bytes), at(Qh, lo * head_bytes),
                                (hi - lo) * head_bytes, cudaMemcpyHostToDevice, xs) != cudaSuccess ||
                cudaEventRecord(q_ready[g], xs) != cudaSuccess)
                return SVGEAR_ERR_CUDA;
        }
        if (cudaMemcpyAsync(w.Kd, Kh, tb, cudaMemcpyHostToDevice, xs) != cudaSuccess ||
            cudaEventRecord(k_ready, xs) != cudaSuccess ||
            cudaMemcpyAsync(w.Vd, Vh, tb, cudaMemcpyHostToDevice, xs) != cudaSuccess ||
            cudaEventRecord(v_ready, xs) != cudaSuccess)
            return SVGEAR_ERR_CUDA;
        // Q, part by part as it arrives
        const size_t cq_row = (size_t)p->Cq * D;
        for (int g = 0; g < GQ; ++g) {
            int lo, hi;
            range(BH, GQ, g, &lo, &hi);
            if (cudaStreamWaitEvent(st, q_ready[g], 0) != cudaSuccess) return SVGEAR_ERR_CUDA;
            if ((s = cluster_heads(at(w.Qd, lo * head_bytes), sub(lo, hi), p->Cq, p->iters,
                                   warm_q ? warm_q + lo * cq_row : nullptr, 2 * p->seed,
                                   (uint64_t)lo, w.labels_q + (size_t)lo * N,
                                   w.perm_q + (size_t)lo * N, w.off_q + (size_t)lo * (p->Cq + 1),
                                   cent_q + lo * cq_row, at(w.Xp_q, lo * head_bytes), w.scratch,
                                   w.scratch_bytes, vst)))
                return s;
        }
        // K, V, value centroids, routing: whole
        if (cudaStreamWaitEvent(st, k_ready, 0) != cudaSuccess) return SVGEAR_ERR_CUDA;
        if ((s = svgear_cluster(w.Kd, dims, p->Ck, p->iters, warm_k, 2 * p->seed + 1, w.labels_k,
                                w.perm_k, w.off_k, cent_k, w.Xp_k, w.scratch, w.scratch_bytes, vst)))
            return s;
        if (cudaStreamWaitEvent(st, v_ready, 0) != cudaSuccess) return SVGEAR_ERR_CUDA;
        if ((s = svgear_permute(w.Vd, w.perm_k, dims, w.Vp, vst))) return s;
        if ((s = svgear_centroids(w.Vp, w.off_k, p->Ck, dims, w.vbar, w.scratch, w.scratch_bytes,
                                  vst)))
            return s;
        if (p->topp > 0.f)
            s = svgear_route_topp(cent_q, w.off_q, p->Cq, cent_k, w.vbar, w.off_k, p->Ck, w.Xp_k,
                                  w.Vp, dims, p->topp, p->scale, w.pair_off, w.pair_kc, nullptr,
                                  nullptr, w.scratch, w.scratch_bytes, vst);
        else
            s = svgear_route(cent_q, w.off_q, p->Cq, cent_k, w.vbar, w.off_k, p->Ck, w.Xp_k, w.Vp,
                             dims, p->density, p->scale, w.pair_off, w.pair_kc, nullptr, w.scratch,
                             w.scratch_bytes, vst);
        if (s) return s;
        if (w.kvar && (s = svgear_key_variance(w.Xp_k, w.off_k, p->Ck, dims, w.kvar, vst)))
            return s;
        // attention part by part; O of each part goes back while the next runs
        // (O lands in Q's device copy: clustering Q was its last reader)
        const size_t ck_row = (size_t)p->Ck * D;
        for (int g = 0; g < GO; ++g) {
            int lo, hi;
            range(BH, GO, g, &lo, &hi);
            const svgear_dims dg = sub(lo, hi);
            if ((s = svgear_attend_var(
                     at(w.Xp_q, lo * head_bytes), at(w.Xp_k, lo * head_bytes),
                     at(w.Vp, lo * head_bytes), dg, N, w.off_q + (size_t)lo * (p->Cq + 1), p->Cq,
                     w.off_k + (size_t)lo * (p->Ck + 1), p->Ck,
                     w.pair_off + (size_t)lo * (p->Cq + 1),
                     w.pair_kc + (size_t)lo * p->Cq * p->Ck, cent_k + lo * ck_row,
                     w.vbar + lo * ck_row, w.kvar ? w.kvar + lo * ck_row : nullptr, p->var_lambda,
                     w.perm_q + (size_t)lo * N, p->scale, at(w.Qd, lo * head_bytes), w.scratch,
                     w.scratch_bytes, vst)))
                return s;
            if (cudaEventRecord(o_ready[g], st) != cudaSuccess ||
                cudaStreamWaitEvent(ds, o_ready[g], 0) != cudaSuccess ||
                cudaMemcpyAsync(at(Oh, lo * head_bytes), at(w.Qd, lo * head_bytes),
                                (hi - lo) * head_bytes, cudaMemcpyDeviceToHost, ds) != cudaSuccess)
                return SVGEAR_ERR_CUDA;
        }
        // the call ends on `st` once O is on the host
        if (cudaEventRecord(done_d2h, ds) != cudaSuccess ||
            cudaStreamWaitEvent(st, done_d2h, 0) != cudaSuccess)
            return SVGEAR_ERR_CUDA;
        return SVGEAR_OK;
    }
};

}  // namespace

extern "C" {

size_t svgear_layer_workspace_bytes(svgear_dims dims, const svgear_layer_params* params,
                                    int32_t host_buffers) {
    if (check_params(dims, params) != SVGEAR_OK) return 0;
    Carve cv(nullptr);
    carve_layer(cv, dims, params, host_buffers != 0);
    return cv.off + kAlign;
}

int svgear_layer(const void* Q, const void* K, const void* V, svgear_dims dims,
                 const svgear_layer_params* params, const float* warm_q, const float* warm_k,
                 void* O, float* cent_q, float* cent_k, void* ws, size_t ws_bytes,
                 void* const* stage_events, void* stream) {
    int s = check_params(dims, params);
    if (s) return s;
    if (!Q || !K || !V || !O || !ws) return SVGEAR_ERR_INVALID_ARG;
    if (ws_bytes < svgear_layer_workspace_bytes(dims, params, 0)) return SVGEAR_ERR_WORKSPACE;
    if (bh_of(dims) == 0) return SVGEAR_OK;
    Carve cv(ws);
    LayerWs w = carve_layer(cv, dims, params, false);
    return run_layer(Q, K, V, dims, params, warm_q, warm_k, O, cent_q, cent_k, w, stage_events,
                     nullptr, static_cast<cudaStream_t>(stream));
}

int svgear_layer_host(const void* Q_host, const void* K_host, const void* V_host,
                      svgear_dims dims, const svgear_layer_params* params, const float* warm_q,
                      const float* warm_k, void* O_host, float* cent_q, float* cent_k, void* ws,
                      size_t ws_bytes, void* stream) {
    int s = check_params(dims, params);
    if (s) return s;
    if (!Q_host || !K_host || !V_host || !O_host || !ws) return SVGEAR_ERR_INVALID_ARG;
    if (ws_bytes < svgear_layer_workspace_bytes(dims, params, 1)) return SVGEAR_ERR_WORKSPACE;
    if (bh_of(dims) == 0) return SVGEAR_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    Carve cv(ws);
    LayerWs w = carve_layer(cv, dims, params, true);
    HostPipeline hp;
    s = hp.run(Q_host, K_host, V_host, dims, params, warm_q, warm_k, O_host, cent_q, cent_k, w,
               st);
    hp.release();
    return s;
}

}  // extern "C"
