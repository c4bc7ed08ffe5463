// w4_debug.cuh -- the in-kernel bounds checks of the W4_DEBUG build.
//
// Built with -DW4_DEBUG, W4_CHECK(cond, status) evaluates cond; when it is
// false it records the failure in the library's device status word and
// yields false, so that the caller skips the access it guards.  A check
// tests the very address expression its access uses.  Where the skipped code
// holds a warp-collective instruction the check is W4_CHECK_WARP (one vote
// for the warp), so that no lane skips it alone.  Nothing
// traps and nothing waits: the context stays usable and the host reads the
// failure with w4_device_status / w4_debug_first_failure.  Without W4_DEBUG
// the macro is the constant true (cond is not evaluated) and costs nothing.
//
// Status word: bit 0 -- a bounded wait ran out; bit 1 -- a bounds check
// failed; bits 2..7 -- the file id of the first failed check (kDbgFile of
// the including file); bits 8..31 -- its source line.
#pragma once

#include <cstdint>

namespace w4 {

#ifdef W4_DEBUG
__device__ __forceinline__ void dbg_fail(unsigned *status, unsigned file, unsigned line) {
    atomicOr(status, 2u);
    // the first failure records its location; a few bounded retries against
    // concurrent changes of the low bits
    unsigned cur = atomicOr(status, 0u);
    for (int i = 0; i < 8 && (cur >> 2) == 0; ++i) {
        const unsigned prev = atomicCAS(status, cur, cur | ((file & 63u) << 2) | (line << 8));
        if (prev == cur) break;
        cur = prev;
    }
}
#define W4_CHECK(cond, status) \
    ((cond) ? true : (::w4::dbg_fail((status), kDbgFile, static_cast<unsigned>(__LINE__)), false))
// The same check voted over the whole (converged) warp: true only if it holds
// in every lane, so that a skip never splits a warp in front of a
// warp-collective instruction (mma.sync, shuffles, votes, .sync.aligned).
#define W4_CHECK_WARP(cond, status) __all_sync(0xffffffffu, W4_CHECK(cond, status))
#else
#define W4_CHECK(cond, status) ((void)sizeof(cond), true)
#define W4_CHECK_WARP(cond, status) ((void)sizeof(cond), true)
#endif

// Bytes of dynamic shared memory of this launch.
__device__ __forceinline__ uint32_t dyn_smem_bytes() {
    uint32_t v;
    asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(v));
    return v;
}

// [addr, addr + bytes) lies inside [base, base + size).
__device__ __forceinline__ bool in_range(uint64_t addr, uint64_t bytes, uint64_t base, uint64_t size) {
    return addr >= base && bytes <= size && addr - base <= size - bytes;
}

}  // namespace w4
