// zha_sync.cuh -- bounded inter-CTA barriers of the persistent decode kernel.
//
// Every barrier is a monotone arrival counter in global memory: a CTA adds 1
// with a release reduction and waits (acquire loads) until the counter reaches
// its own epoch x the number of participants.  One L2 round trip per arrival,
// no reset between barriers.  The counters are cleared by the last CTA to
// leave the kernel (exit counter), so each launch starts from zero.  Every
// wait is bounded by a clock budget (Decode::wait_budget, about one second
// unless a test lowers it); on expiry the CTA records
// ZHA_TIMEOUT_CODE, raises the abort word and returns false, and every other
// waiter returns false as soon as it sees the abort word.
//
// Layout of the sync words (uint32, zeroed at context creation):
//   [0, h_kv)   team counters, one per KV head
//   h_kv        grid counter
//   h_kv + 1    exit counter
//   h_kv + 2    abort word
#pragma once

#include "zha_device.cuh"
#include "zha_internal.cuh"
#include "zha_tma.cuh"

namespace zha {

__device__ __forceinline__ unsigned ld_relaxed_u32(const unsigned *p) {
    unsigned v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }

__device__ __forceinline__ void red_release_add_u32(unsigned *p, unsigned v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Thread-level arrive-and-wait on a counter; false on abort or timeout.
// `budget`: clock cycles the wait may take (Decode::wait_budget).
__device__ __noinline__ bool counter_arrive_wait(unsigned *ctr, unsigned target, unsigned *abortw, int32_t *status,
                                                 long long budget) {
    red_release_add_u32(ctr, 1u);
    const long long t0 = clock64();
    for (;;) {
        // two independent relaxed polls per round trip; the fence after the
        // counter is seen makes the pair an acquire of every arrival
        const unsigned c = ld_relaxed_u32(ctr), ab = ld_relaxed_u32(abortw);
        if (c >= target) {
            fence_acq_rel_gpu();
            return true;
        }
        if (ab) return false;
        if (clock64() - t0 > budget) {
            set_status(status, ZHA_TIMEOUT_CODE);
            atomicExch(abortw, 1u);
            return false;
        }
    }
}

// Barrier among the CTAs of one team (or of the grid), entered by the 256
// routing threads (named barrier 1) of each CTA.  `epoch` counts the
// barriers this CTA has passed on this counter.
__device__ __forceinline__ bool team_barrier(unsigned *ctr, int members, unsigned &epoch, unsigned *abortw,
                                             int32_t *status, int *s_flag, long long budget) {
    gsync();
    if (threadIdx.x == 0) {
        epoch += 1u;
        *s_flag = counter_arrive_wait(ctr, epoch * (unsigned)members, abortw, status, budget) ? 1 : 0;
    }
    gsync();
    return *s_flag != 0;
}

// The same for all threads of the CTA (__syncthreads).
__device__ __forceinline__ bool grid_barrier(unsigned *ctr, int members, unsigned &epoch, unsigned *abortw,
                                             int32_t *status, int *s_flag, long long budget) {
    __syncthreads();
    if (threadIdx.x == 0) {
        epoch += 1u;
        *s_flag = counter_arrive_wait(ctr, epoch * (unsigned)members, abortw, status, budget) ? 1 : 0;
    }
    __syncthreads();
    return *s_flag != 0;
}

// Leave the kernel: the last CTA out clears every counter and the abort word
// (nothing else can be waiting on them then).  Called by all threads.
__device__ __forceinline__ void kernel_exit(unsigned *words, int n_words, int exit_index) {
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const unsigned prev = atomicAdd(words + exit_index, 1u);
        if (prev == gridDim.x - 1) {
            for (int i = 0; i < n_words; ++i) atomicExch(words + i, 0u);
            __threadfence();
        }
    }
}

}  // namespace zha
