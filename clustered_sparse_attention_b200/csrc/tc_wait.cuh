// tc_wait.cuh -- bounded mbarrier waits shared by the tcgen05 kernels.
//
// Every wait gives up after kWaitTimeoutNs of %globaltimer (or after
// kMaxSpins polls, should the timer not advance), or at once when this CTA
// (its shared abort flag) or any CTA of the launch (the device status word)
// has already given up.  err[0] is the status word; the first expired wait
// records where it was (err[1] = site * 65536 + index) and which CTA
// (err[2] = blockIdx.y * 65536 + blockIdx.x).  A kernel that gives up drains
// what it issued, keeps its TMEM allocated if an MMA may still be running
// (and then sets the device's tensor-memory-lost word, guard.cu), and
// returns; the host reads the status word.
#pragma once

#include "common.cuh"
#include "tc_ptx.cuh"

namespace svgear {
namespace tc {

constexpr uint64_t kWaitTimeoutNs = 1000000000ull;   // 1 s; a tile takes microseconds
constexpr uint32_t kMaxSpins = 1u << 30;              // backstop: tens of seconds of polls

// Wait sites outside the kernels' own numbering (err[1] >> 16).
constexpr int kSiteSelftest = 60;   // svgear_selftest_wait
constexpr int kSiteTmemLost = 61;   // refused to start: the device's TMEM was lost earlier

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                         int* err, int where,
                                         uint64_t timeout_ns = kWaitTimeoutNs) {
    const uint32_t b = smem_u32(bar);
    if (mbar_try_wait(b, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    volatile int* gerr = err;
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(b, parity)) return true;
        if ((it & 63) != 0) continue;   // check the abort flags and the clock now and then
        if (*abort_flag || *gerr) {
            *abort_flag = 1;
            return false;
        }
        if (global_timer_ns() - t0 > timeout_ns || it >= kMaxSpins) {
            *abort_flag = 1;
            if (atomicCAS(err, 0, SVGEAR_ERR_TIMEOUT) == 0) {
                err[1] = where;
                err[2] = (int)(blockIdx.y * 65536 + blockIdx.x);
            }
            return false;
        }
    }
}

// The device's tensor-memory-lost word (guard.cu): set by a kernel that kept
// its TMEM columns because an MMA it issued may still have been running.
__device__ __forceinline__ void mark_tmem_lost(int* lost) {
    atomicExch(lost, 1);
    __threadfence();
}

// Called by every thread of a tcgen05 kernel before it allocates TMEM: true
// (the same answer in every thread) when the kernel must return at once,
// because another CTA of the launch already gave up (err set) or the
// device's TMEM was lost earlier; the latter is recorded in the status word
// as SVGEAR_ERR_TMEM_LOST.  One thread reads, so the CTA leaves together.
__device__ __forceinline__ bool refuse_start(const int* lost, int* err) {
    int stop = 0;
    if (threadIdx.x == 0) {
        if (*(volatile const int*)lost != 0) {
            stop = 1;
            if (atomicCAS(err, 0, SVGEAR_ERR_TMEM_LOST) == 0) {
                err[1] = kSiteTmemLost << 16;
                err[2] = (int)(blockIdx.y * 65536 + blockIdx.x);
            }
        } else if (*(volatile int*)err != 0) {
            stop = 1;
        }
    }
    return __syncthreads_or(stop) != 0;
}

// One lane polls, the whole warp gets the same answer, so warps that run
// .sync.aligned TMEM instructions or reach a CTA barrier stay converged.
__device__ __forceinline__ bool warp_wait_bar(uint64_t* bar, uint32_t parity,
                                              volatile int* abort_flag, int* err, int where) {
    int ok = 0;
    if ((threadIdx.x & 31) == 0) ok = wait_bar(bar, parity, abort_flag, err, where) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok != 0;
}

}  // namespace tc
}  // namespace svgear
