// peer.cuh -- 64-bit relaxed accesses at system scope, for words that other
// GPUs write over NVLink (or read).  A naturally aligned 64-bit access is
// single-copy atomic: a reader sees either the old word or the new one.
#pragma once

#include <stdint.h>

namespace mlra {
namespace peer {

__device__ __forceinline__ void st_relaxed_sys_u64(uint64_t* p, uint64_t v) {
    asm volatile("st.relaxed.sys.global.u64 [%0], %1;" :: "l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ uint64_t ld_relaxed_sys_u64(const uint64_t* p) {
    uint64_t v;
    asm volatile("ld.relaxed.sys.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

}  // namespace peer
}  // namespace mlra
