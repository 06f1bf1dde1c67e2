// noalloc.cu -- the label sort without a caller-provided workspace.
//
// Some callers cannot hand this library any scratch memory: a host framework
// whose memory planner owns every device byte and forbids side allocations,
// a real-time loop where cudaMalloc (slow and synchronising) is banned once
// running, or a plugin interface that passes an operator only its input and
// output buffers.  svgear_label_sort_noalloc serves them: its scratch (the
// per-block label histograms of the counting sort) lives in the fixed array
// below, which every GPU that loads the library keeps until the process
// exits.  Nothing here calls cudaMalloc, cudaFree or an allocating routine.
#include "common.cuh"
#include "ctx_cache.h"
#include "launchers.h"

namespace {

// File-scope scratch: block histograms [B*H][ceil(N/1024)][C] of int32.
static __device__ __align__(256) int32_t g_sort_scratch[SVGEAR_NOALLOC_SORT_SCRATCH_INTS];

// In host code `g_sort_scratch` names a host-side stand-in, not device memory,
// so the kernels get the device address, looked up once per CUDA context (a
// device reset makes a new context, whose first call looks it up again).
svgear::SymbolAddressCache g_scratch_addr;

int scratch_on_current_device(int32_t** out) {
    void* p = nullptr;
    const int s = g_scratch_addr.get(g_sort_scratch, &p);
    *out = static_cast<int32_t*>(p);
    return s;
}

}  // namespace

extern "C" int svgear_label_sort_noalloc(const int32_t* labels, svgear_dims dims, int32_t C,
                                         int32_t* perm, int32_t* offsets, void* stream) {
    if (dims.B < 0 || dims.H < 0 || dims.N < 1) return SVGEAR_ERR_INVALID_ARG;
    const size_t BH = (size_t)dims.B * (size_t)dims.H;
    if (BH > 65535) return SVGEAR_ERR_UNSUPPORTED;
    if (C < 1 || C > dims.N) return SVGEAR_ERR_INVALID_ARG;
    if (C > SVGEAR_MAX_CLUSTERS) return SVGEAR_ERR_UNSUPPORTED;
    if (!labels || !perm || !offsets) return SVGEAR_ERR_INVALID_ARG;
    const size_t need = BH * (size_t)svgear::ceil_div(dims.N, svgear::kSortTokens) * (size_t)C;
    if (need > (size_t)SVGEAR_NOALLOC_SORT_SCRATCH_INTS) return SVGEAR_ERR_SCRATCH_LIMIT;
    if (BH == 0) return SVGEAR_OK;
    int32_t* hist = nullptr;
    const int s = scratch_on_current_device(&hist);
    if (s != SVGEAR_OK) return s;
    // The histogram pass overwrites every entry the later passes read, so the
    // previous call's contents need no clearing.
    return svgear::launch_label_sort(labels, (int)BH, dims.N, C, perm, offsets, hist,
                                     static_cast<cudaStream_t>(stream));
}
