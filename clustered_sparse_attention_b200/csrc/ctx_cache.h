// ctx_cache.h -- device addresses of file-scope __device__ variables, looked
// up once per CUDA context.
//
// In host code the name of a __device__ variable is a host-side stand-in, not
// a device address; cudaGetSymbolAddress gives the address inside the current
// context.  A context is identified by cuCtxGetId, which is unique over the
// life of the process, so an address looked up before a device reset (which
// destroys the primary context and with it the module that holds the
// variable) is never handed out afterwards: the first call in the new context
// looks the address up again.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <mutex>
#include <vector>

#include "svgear.h"

namespace svgear {

class SymbolAddressCache {
public:
    // *out = device address of `symbol` in the current context.
    template <typename T>
    int get(const T& symbol, void** out) {
        unsigned long long id = 0;
        const bool have_id = current_id(&id);
        if (have_id) {
            std::lock_guard<std::mutex> lock(mu_);
            for (const Entry& e : entries_)
                if (e.ctx_id == id) {
                    *out = e.addr;
                    return SVGEAR_OK;
                }
        }
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, symbol) != cudaSuccess || p == nullptr) return SVGEAR_ERR_CUDA;
        // the lookup made the device's primary context current if none was
        if (have_id || current_id(&id)) {
            std::lock_guard<std::mutex> lock(mu_);
            entries_.push_back(Entry{id, p});
        }
        *out = p;
        return SVGEAR_OK;
    }

    // Unique id of the current context; false when no context is current.
    // The driver calls come through the runtime's entry-point table, so the
    // library does not link against libcuda.
    static bool current_id(unsigned long long* id) {
        static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
        static PFN_cuCtxGetId_v12000 get_id = nullptr;
        static std::once_flag once;
        std::call_once(once, [] {
            void* p = nullptr;
            cudaDriverEntryPointQueryResult q;
            if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
                q == cudaDriverEntryPointSuccess)
                get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
            p = nullptr;
            if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
                q == cudaDriverEntryPointSuccess)
                get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
        });
        if (!get_current || !get_id) return false;
        CUcontext ctx = nullptr;
        if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
        return get_id(ctx, id) == CUDA_SUCCESS;
    }

private:
    struct Entry {
        unsigned long long ctx_id;
        void* addr;
    };
    std::mutex mu_;
    std::vector<Entry> entries_;
};

}  // namespace svgear
