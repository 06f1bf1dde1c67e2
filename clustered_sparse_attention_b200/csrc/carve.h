// carve.h -- bump allocation over a caller's workspace (internal).
#pragma once

#include <stddef.h>

namespace svgear {

constexpr size_t kAlign = 256;

// Bump allocator over the caller's workspace; with base == nullptr it only
// measures, so sizing and carving share one description of the layout.
struct Carve {
    char* base;
    size_t off = 0;
    explicit Carve(void* b) : base(static_cast<char*>(b)) {}
    template <typename T> T* take(size_t count) {
        off = (off + kAlign - 1) / kAlign * kAlign;
        T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
        off += sizeof(T) * count;
        return p;
    }
};

}  // namespace svgear
