// zha_attend.cu -- dense flash-decode over the whole cache (sm_100a): the
// comparison kernel, exact softmax attention of every query head over all
// rows 0 .. N-1, through the same bulk-copy pipeline as the routed attention.
// The last CTA to finish a KV head's stages (fence + ticket) merges its
// partials.
#include "zha_attend.cuh"

namespace zha {

template <typename KT, int HD, int G>
__global__ void __launch_bounds__(A_THREADS, 1) k_dense(const __grid_constant__ Decode a) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ StageMap map;
    __shared__ int s_last[64];
    const int warp = threadIdx.x >> 5;
    const int h_kv = a.nvk, nb = gridDim.x, b = blockIdx.x;
    stage_map_init<true, StageCfg<KT, HD>::TT>(a, map);
    attn_stages<KT, HD, G, true>(a, map, smem, b, nb);
    __threadfence();
    __syncthreads();
    if (threadIdx.x < h_kv) {
        const int kh = threadIdx.x;
        int bf, bl;
        map.ctas(kh, nb, bf, bl);
        int last = 0;
        if (bl >= 0 && b >= bf && b <= bl) {
            const unsigned tk = atomicAdd(a.ticket + kh, 1u);
            last = (tk == (unsigned)(bl - bf));
            if (last) a.ticket[kh] = 0u;
        }
        s_last[kh] = last;
    }
    __syncthreads();
    for (int kh = 0; kh < h_kv; ++kh) {
        if (!s_last[kh]) continue;
        __threadfence();
        int bf, bl;
        map.ctas(kh, nb, bf, bl);
        if (warp < ACW) combine_kvh<KT, HD, G>(a, map, kh, bf, bl + 1, false, reinterpret_cast<float *>(smem));
        __syncthreads();
    }
}

template <typename KT, int HD, int G>
static cudaError_t dense_impl(const Decode &dc, int n_cta, cudaStream_t s) {
    const size_t smem = ASmem<KT, HD, G>::bytes;
    static PerDeviceMax<> attr;
    const cudaError_t err = allow_smem(k_dense<KT, HD, G>, smem, attr);
    if (err != cudaSuccess) return err;
    k_dense<KT, HD, G><<<n_cta, A_THREADS, smem, s>>>(dc);
    return cudaGetLastError();
}

cudaError_t launch_dense(const Decode &dc, int n_cta, cudaStream_t s) {
    const Tree &t = dc.t;
    if (t.kv_dtype == 1) {
        if (t.d == 128 && t.G == 4) return dense_impl<uint16_t, 128, 4>(dc, n_cta, s);
        if (t.d == 128 && t.G == 1) return dense_impl<uint16_t, 128, 1>(dc, n_cta, s);
        if (t.d == 64 && t.G == 4) return dense_impl<uint16_t, 64, 4>(dc, n_cta, s);
        if (t.d == 64 && t.G == 1) return dense_impl<uint16_t, 64, 1>(dc, n_cta, s);
    } else {
        if (t.d == 128 && t.G == 4) return dense_impl<float, 128, 4>(dc, n_cta, s);
        if (t.d == 128 && t.G == 1) return dense_impl<float, 128, 1>(dc, n_cta, s);
        if (t.d == 64 && t.G == 4) return dense_impl<float, 64, 4>(dc, n_cta, s);
        if (t.d == 64 && t.G == 1) return dense_impl<float, 64, 1>(dc, n_cta, s);
    }
    return cudaErrorInvalidValue;
}

bool compiled_combo(int kv_dtype, int d, int R, int G, int router) {
    if (router == 1 && (kv_dtype != 1 || d != 128)) return false;  // bf16 router: bf16 caches, d = 128
    return (d == 64 || d == 128) && (R == 1 || R == 16) && (G == 1 || G == 4);
}

}  // namespace zha
