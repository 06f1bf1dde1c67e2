// guard.cu -- the tensor-memory guard shared by the tcgen05 kernels, and the
// self-test of the library's bounded device wait.
//
// A tcgen05 kernel that gives up on a wait while an MMA it issued may still be
// running cannot release its tensor memory (TMEM): freeing columns an MMA
// still writes is undefined, so the kernel keeps them allocated.  On that SM a
// later tcgen05.alloc would then wait for good.  So the kernel also sets
// g_tmem_lost, one word per device that no call clears: every tcgen05 kernel
// reads it before allocating and returns SVGEAR_ERR_TMEM_LOST instead, and
// svgear_device_status latches it on the host, after which the tensor-core
// entry points return that status without launching.  The loss lasts as long
// as the CUDA context (the process, or until a device reset).
#include <mutex>
#include <vector>

#include "common.cuh"
#include "ctx_cache.h"
#include "launchers.h"
#include "tc_ptx.cuh"
#include "tc_wait.cuh"

namespace svgear {
namespace {

static __device__ int g_tmem_lost;

SymbolAddressCache g_lost_addr;

// Host latch: ids of the contexts whose lost word was seen set.
std::mutex g_latch_mu;
std::vector<unsigned long long> g_latched;

// One CTA, one thread: wait on an mbarrier that has one expected arrival,
// made first when `arrive` is set; otherwise nothing arrives and the bounded
// wait gives up after timeout_ns.
__global__ void wait_selftest_kernel(int arrive, unsigned long long timeout_ns, int mark_lost,
                                     int* lost, int* err) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x != 0) return;
    tc::mbar_init(tc::smem_u32(&bar), 1);
    abort_flag = 0;
    tc::mbar_init_fence();
    if (arrive) tc::mbar_arrive(tc::smem_u32(&bar));
    const bool ok = tc::wait_bar(&bar, 0, &abort_flag, err, (tc::kSiteSelftest << 16), timeout_ns);
    if (!ok && mark_lost) tc::mark_tmem_lost(lost);
}

}  // namespace

int tmem_lost_word(int** out) {
    void* p = nullptr;
    const int s = g_lost_addr.get(g_tmem_lost, &p);
    *out = static_cast<int*>(p);
    return s;
}

bool tmem_lost_latched() {
    unsigned long long id = 0;
    if (!SymbolAddressCache::current_id(&id)) return false;
    std::lock_guard<std::mutex> lock(g_latch_mu);
    for (unsigned long long x : g_latched)
        if (x == id) return true;
    return false;
}

static void latch_tmem_lost() {
    unsigned long long id = 0;
    if (!SymbolAddressCache::current_id(&id)) return;
    std::lock_guard<std::mutex> lock(g_latch_mu);
    for (unsigned long long x : g_latched)
        if (x == id) return;
    g_latched.push_back(id);
}

}  // namespace svgear

using namespace svgear;

extern "C" {

int svgear_device_status(const void* ws, size_t ws_bytes, int32_t* status, void* stream) {
    if (!ws || !status || ws_bytes < 4 * sizeof(int)) return SVGEAR_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int* lost = nullptr;
    int s = tmem_lost_word(&lost);
    if (s != SVGEAR_OK) return s;
    int32_t words[4] = {0, 0, 0, 0};
    int32_t lost_word = 0;
    if (cudaMemcpyAsync(words, ws, sizeof(words), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaMemcpyAsync(&lost_word, lost, sizeof(int32_t), cudaMemcpyDeviceToHost, st) !=
            cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return SVGEAR_ERR_CUDA;
    status[0] = words[0];
    status[1] = words[1];
    status[2] = words[2];
    status[3] = lost_word != 0 ? 1 : 0;
    if (lost_word) latch_tmem_lost();
    return SVGEAR_OK;
}

int svgear_attend_status(const void* ws, size_t ws_bytes, int32_t* status, void* stream) {
    return svgear_device_status(ws, ws_bytes, status, stream);
}

int svgear_selftest_wait(void* ws, size_t ws_bytes, int32_t arrive, int32_t timeout_us,
                         int32_t mark_lost, void* stream) {
    if (!ws || ws_bytes < 4 * sizeof(int)) return SVGEAR_ERR_INVALID_ARG;
    if (timeout_us < 1 || timeout_us > 10000000) return SVGEAR_ERR_INVALID_ARG;
    if ((arrive != 0 && arrive != 1) || (mark_lost != 0 && mark_lost != 1))
        return SVGEAR_ERR_INVALID_ARG;
    int* lost = nullptr;
    int s = tmem_lost_word(&lost);
    if (s != SVGEAR_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int* err = static_cast<int*>(ws);
    if (cudaMemsetAsync(err, 0, 4 * sizeof(int), st) != cudaSuccess) return SVGEAR_ERR_CUDA;
    wait_selftest_kernel<<<1, 32, 0, st>>>(arrive, (unsigned long long)timeout_us * 1000ull,
                                           mark_lost, lost, err);
    count_launches(1);
    SVGEAR_LAUNCH_CHECK();
    return SVGEAR_OK;
}

}  // extern "C"
