// 32-byte global loads and stores (sm_100 and later): one instruction moves 8 words, half the
// memory instructions of 16-byte vectors for the row copies and gathers of the HBM-bound kernels.
#pragma once

#include <stdint.h>

namespace moe {

// 32-byte vectors (sm_100 and later): one instruction moves 8 words.  Addresses 32-byte aligned.
struct Vec32 {
    uint32_t w[8];
};

// read-only (non-coherent) path, for data no kernel writes while it runs
__device__ __forceinline__ Vec32 ld_nc_v8(const void* p) {
    Vec32 v;
    asm volatile("ld.global.nc.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(v.w[0]), "=r"(v.w[1]), "=r"(v.w[2]), "=r"(v.w[3]), "=r"(v.w[4]), "=r"(v.w[5]), "=r"(v.w[6]),
                   "=r"(v.w[7])
                 : "l"(p));
    return v;
}

__device__ __forceinline__ void st_v8(void* p, const Vec32& v) {
    asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(v.w[0]), "r"(v.w[1]), "r"(v.w[2]),
                 "r"(v.w[3]), "r"(v.w[4]), "r"(v.w[5]), "r"(v.w[6]), "r"(v.w[7])
                 : "memory");
}

}  // namespace moe
