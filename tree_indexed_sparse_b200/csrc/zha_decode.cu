// zha_decode.cu -- one decoded token for every query head, in one persistent
// cooperative kernel (sm_100a): every routing level, then the routed
// attention, with bounded grid barriers between the phases.
//
// Routing ("ZHA 用树形稀疏注意力改造现有大模型", section "稀疏注意力为什么还会被索引拖慢":
// score the top nodes, keep the smallest set whose estimated mass reaches p,
// expand only their children, repeat down to the raw entries; "Zyphra
// 分层注意力（ZHA）…", section "机制拆解：树形索引如何高效筛选长上下文"):
//   level D .. 1:
//     a frontier small enough for one SM (<= SMALL_BYTES of summaries per KV
//     head) is scored and cut by the CTA that owns its KV head, with no
//     fan-in; a larger one is scored by every CTA of the grid (each KV head
//     gets gridDim/h_kv CTAs), then, after a grid barrier, cut by its owner;
//     a grid barrier ends the level.
//   attention over the kept leaves plus the sink token, split over every CTA
//   (zha_attend.cuh), a grid barrier, and the owner CTAs merge the partials.
// The grid is one CTA per SM, launched cooperatively so that the barriers
// cannot deadlock; every barrier wait is bounded by a clock budget, after
// which the kernel records ZHA_ERR_TIMEOUT, raises a shared abort flag and
// returns.
#include "zha_attend.cuh"
#include "zha_route.cuh"
#include "zha_select.cuh"

namespace zha {

constexpr int64_t SMALL_BYTES = 256 * 1024;

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Grid barrier over all CTAs (cooperative launch: all are resident).  gbar[0]
// counts arrivals, gbar[1] is the generation, gbar[2] the abort flag.
__device__ __noinline__ bool grid_sync(const Decode &a) {
    __shared__ int s_ok;
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned *count = a.gbar, *gen = a.gbar + 1, *abortf = a.gbar + 2;
        const unsigned g = ld_acquire_u32(gen);
        __threadfence();
        int ok = 1;
        if (atomicAdd(count, 1u) == gridDim.x - 1) {
            atomicExch(count, 0u);
            __threadfence();
            atomicAdd(gen, 1u);
        } else {
            const long long t0 = clock64();
            while (ld_acquire_u32(gen) == g) {
                if (ld_acquire_u32(abortf)) { ok = 0; break; }
                if (clock64() - t0 > WAIT_BUDGET_CYCLES) {
                    set_status(a.status, ZHA_TIMEOUT_CODE);
                    atomicExch(abortf, 1u);
                    ok = 0;
                    break;
                }
                __nanosleep(32);
            }
        }
        __threadfence();
        s_ok = ok && !ld_acquire_u32(abortf);
    }
    __syncthreads();
    return s_ok != 0;
}

__device__ __forceinline__ void stamp(const Decode &a, int i) {
    if (a.phase_ns && blockIdx.x == 0 && threadIdx.x == 0) {
        unsigned long long t;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
        a.phase_ns[i] = (int64_t)t;
    }
}

template <typename KT, int HD, int R, int G>
__global__ void __launch_bounds__(A_THREADS, 1) k_decode(const __grid_constant__ Decode a) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ StageMap map;
    const int warp = threadIdx.x >> 5;
    const int nb = gridDim.x, b = blockIdx.x;
    const int h_kv = a.t.h_kv;
    const int nbk = nb / h_kv;  // CTAs per KV head when a level is scored by the whole grid
    float *wsm = reinterpret_cast<float *>(smem);
    stamp(a, 0);
    for (int l = a.t.D; l >= 1; --l) {
        int64_t smax = 0;
        for (int kh = 0; kh < h_kv; ++kh) smax = max(smax, frontier_size(a, l, kh));
        const bool small = smax * (int64_t)(R * HD * 4) <= SMALL_BYTES;
        if (small) {
            if (b < h_kv && warp < ACW) {
                const int64_t S = frontier_size(a, l, b);
                route_score<HD, R, G>(a, l, b, 0, 1, S, wsm);
                select_kvh<HD, R, G>(a, l, b, S, 1, smem);
            }
        } else {
            if (b < nbk * h_kv && warp < ACW)
                route_score<HD, R, G>(a, l, b % h_kv, b / h_kv, nbk, frontier_size(a, l, b % h_kv), wsm);
            if (!grid_sync(a)) return;
            if (b < h_kv && warp < ACW) select_kvh<HD, R, G>(a, l, b, frontier_size(a, l, b), nbk, smem);
        }
        if (!grid_sync(a)) return;
        stamp(a, a.t.D - l + 1);
    }
    if (threadIdx.x == 0) stage_map_init<false>(a, map);
    __syncthreads();
    attn_stages<KT, HD, G, false>(a, map, smem, b, nb);
    if (!grid_sync(a)) return;
    stamp(a, a.t.D + 1);
    if (b < h_kv && warp < ACW) {
        int bf, bl;
        map.ctas(b, nb, bf, bl);
        combine_kvh<KT, HD, G>(a, b, bf, bl + 1, true, reinterpret_cast<float *>(smem));
    }
    stamp(a, a.t.D + 2);
}

template <typename KT, int HD, int R, int G>
static cudaError_t decode_impl(const Decode &dc, int n_cta, cudaStream_t s) {
    const size_t smem = std::max(SelectSmem<G>::bytes, ASmem<KT, HD, G>::bytes);
    static size_t attr = 0;
    if (smem > attr) {
        cudaError_t err =
            cudaFuncSetAttribute(k_decode<KT, HD, R, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err != cudaSuccess) return err;
        attr = smem;
    }
    Decode arg = dc;
    void *args[] = {&arg};
    return cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(k_decode<KT, HD, R, G>), dim3(n_cta),
                                       dim3(A_THREADS), args, smem, s);
}

template <typename KT, int HD, int R, int G>
static int decode_occupancy() {
    const size_t smem = std::max(SelectSmem<G>::bytes, ASmem<KT, HD, G>::bytes);
    static size_t attr = 0;
    if (smem > attr) {
        if (cudaFuncSetAttribute(k_decode<KT, HD, R, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
            return 0;
        attr = smem;
    }
    int blocks = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, k_decode<KT, HD, R, G>, A_THREADS, smem) != cudaSuccess)
        return 0;
    return blocks;
}

#define ZHA_DECODE_DISPATCH(FN, ...)                                                         \
    do {                                                                                     \
        const Tree &t = dc.t;                                                                \
        if (t.kv_dtype == 1) {                                                               \
            if (t.d == 128 && t.R == 16 && t.G == 4) return FN<uint16_t, 128, 16, 4>(__VA_ARGS__); \
            if (t.d == 128 && t.R == 1 && t.G == 4) return FN<uint16_t, 128, 1, 4>(__VA_ARGS__);   \
            if (t.d == 128 && t.R == 16 && t.G == 1) return FN<uint16_t, 128, 16, 1>(__VA_ARGS__); \
            if (t.d == 128 && t.R == 1 && t.G == 1) return FN<uint16_t, 128, 1, 1>(__VA_ARGS__);   \
            if (t.d == 64 && t.R == 16 && t.G == 4) return FN<uint16_t, 64, 16, 4>(__VA_ARGS__);   \
            if (t.d == 64 && t.R == 1 && t.G == 4) return FN<uint16_t, 64, 1, 4>(__VA_ARGS__);     \
            if (t.d == 64 && t.R == 16 && t.G == 1) return FN<uint16_t, 64, 16, 1>(__VA_ARGS__);   \
            if (t.d == 64 && t.R == 1 && t.G == 1) return FN<uint16_t, 64, 1, 1>(__VA_ARGS__);     \
        } else {                                                                             \
            if (t.d == 128 && t.R == 16 && t.G == 4) return FN<float, 128, 16, 4>(__VA_ARGS__);    \
            if (t.d == 128 && t.R == 1 && t.G == 4) return FN<float, 128, 1, 4>(__VA_ARGS__);      \
            if (t.d == 128 && t.R == 16 && t.G == 1) return FN<float, 128, 16, 1>(__VA_ARGS__);    \
            if (t.d == 128 && t.R == 1 && t.G == 1) return FN<float, 128, 1, 1>(__VA_ARGS__);      \
            if (t.d == 64 && t.R == 16 && t.G == 4) return FN<float, 64, 16, 4>(__VA_ARGS__);      \
            if (t.d == 64 && t.R == 1 && t.G == 4) return FN<float, 64, 1, 4>(__VA_ARGS__);        \
            if (t.d == 64 && t.R == 16 && t.G == 1) return FN<float, 64, 16, 1>(__VA_ARGS__);      \
            if (t.d == 64 && t.R == 1 && t.G == 1) return FN<float, 64, 1, 1>(__VA_ARGS__);        \
        }                                                                                    \
    } while (0)

cudaError_t launch_decode(const Decode &dc, int n_cta, cudaStream_t s) {
    ZHA_DECODE_DISPATCH(decode_impl, dc, n_cta, s);
    return cudaErrorInvalidValue;
}

int decode_blocks_per_sm(const Decode &dc) {
    ZHA_DECODE_DISPATCH(decode_occupancy);
    return 0;
}

}  // namespace zha
