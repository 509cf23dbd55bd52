// zha_static.cu -- dense decode straight from a KV cache with no context and no
// workspace: the split partials and merge tickets of k_dense live in a fixed
// scratch array that the library's device image carries.
//
// Which callers need this: layers that keep plain dense attention (no tree)
// inside a serving engine that reserves all of its device memory up front and
// forbids allocation while it serves.  Such a caller holds the KV cache and
// the query/output buffers but has no workspace to give and may not allocate
// one, so the library supplies the scratch itself, from static storage that
// exists as soon as the module is loaded.
//
// Set-up: the first call on a device looks up the scratch's address there,
// and, under CUDA's default lazy module loading, loading the module for that
// device is what reserves the scratch (and the kernel code).  Callers make
// that first call while setting up, before they serve and before any stream
// capture; from then on a call allocates nothing.
//
// Limits: one call at a time per device.  Every call uses the same scratch, so
// two calls in flight together (other streams, other host threads) race on it
// and corrupt each other's outputs.  Configurations whose partials do not fit
// in ZHA_STATIC_SCRATCH_BYTES are rejected.
#include <algorithm>
#include <cmath>
#include <mutex>

#include "../../include/zha.h"
#include "zha_internal.cuh"
#include "zha_tma.cuh"

using namespace zha;

static __device__ __align__(256) unsigned char g_dense_scratch[ZHA_STATIC_SCRATCH_BYTES];

namespace {

constexpr int DEV_MAX = 64;
constexpr int STATIC_CTA_CAP = SEG_CAP;  // the context path's cap on attention CTAs

struct DevScratch {
    unsigned char *ptr = nullptr;  // device address of g_dense_scratch on this device
    int n_sm = 0;
};

std::mutex g_mu;
DevScratch g_dev[DEV_MAX];

int64_t align256(int64_t x) { return (x + 255) / 256 * 256; }

// Once per device, with that device current: the scratch's device address and
// the SM count.  The first call on a device does this.
int device_scratch(DevScratch &out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ZHA_ERR_CUDA;
    if (dev < 0 || dev >= DEV_MAX) return ZHA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mu);
    DevScratch &d = g_dev[dev];
    if (!d.ptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_dense_scratch) != cudaSuccess || !p) return ZHA_ERR_CUDA;
        int n_sm = 0;
        if (cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n_sm < 1)
            return ZHA_ERR_CUDA;
        d.n_sm = n_sm;
        d.ptr = static_cast<unsigned char *>(p);
    }
    out = d;
    return ZHA_OK;
}

}  // namespace

extern "C" {

int zha_dense_decode_static(const zha_config *cfg, const void *d_K, const void *d_V, int64_t n_tokens,
                            const float *d_q, float *d_out, int32_t *d_status, void *stream) {
    if (!cfg || !d_K || !d_V || !d_q || !d_out || !d_status) return ZHA_ERR_BAD_ARG;
    if (cfg->h_kv < 1 || cfg->h_kv > 64 || cfg->h_q < cfg->h_kv || cfg->h_q % cfg->h_kv) return ZHA_ERR_BAD_ARG;
    if (cfg->kv_dtype != ZHA_F32 && cfg->kv_dtype != ZHA_BF16) return ZHA_ERR_BAD_ARG;
    if (cfg->capacity_tokens < 1 || cfg->capacity_tokens > (int64_t)0x7fffffff) return ZHA_ERR_BAD_ARG;
    if (n_tokens < 1 || n_tokens > cfg->capacity_tokens) return ZHA_ERR_BAD_ARG;
    if (((reinterpret_cast<uintptr_t>(d_K) | reinterpret_cast<uintptr_t>(d_V) | reinterpret_cast<uintptr_t>(d_q) |
          reinterpret_cast<uintptr_t>(d_out)) & 15u) ||
        (reinterpret_cast<uintptr_t>(d_status) & 3u))
        return ZHA_ERR_BAD_ARG;
    const int G = cfg->h_q / cfg->h_kv;
    if (!compiled_combo(cfg->kv_dtype, cfg->d, 1, G, 0)) return ZHA_ERR_UNSUPPORTED;

    DevScratch ds;
    const int rc = device_scratch(ds);
    if (rc != ZHA_OK) return rc;
    // the same grid as the context path: one CTA per SM
    const int n_cta = std::min(STATIC_CTA_CAP, ds.n_sm);
    const int64_t part_bytes = align256((int64_t)n_cta * cfg->h_q * (cfg->d + 4) * 4);
    const int64_t ticket_bytes = (int64_t)cfg->h_kv * 4;
    if (part_bytes + ticket_bytes > (int64_t)ZHA_STATIC_SCRATCH_BYTES) return ZHA_ERR_CAPACITY;

    Decode dc{};
    Tree &t = dc.t;
    t.h_kv = cfg->h_kv;
    t.h_q = cfg->h_q;
    t.G = G;
    t.d = cfg->d;
    t.R = 1;
    t.c = 1;
    t.D = 1;
    t.kv_dtype = cfg->kv_dtype;
    t.c_log2 = -1;
    t.kv_cap = cfg->capacity_tokens;
    t.n_tokens = n_tokens;
    t.K = d_K;
    t.V = d_V;
    t.scale = (float)(1.0 / std::sqrt((double)cfg->d));
    dc.nvk = cfg->h_kv;
    dc.q = d_q;
    dc.out = d_out;
    dc.part = reinterpret_cast<float *>(ds.ptr);
    dc.part_cap = n_cta;
    dc.ticket = reinterpret_cast<uint32_t *>(ds.ptr + part_bytes);
    dc.status = d_status;
    dc.wait_budget = WAIT_BUDGET_CYCLES;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the merge tickets must start at zero (a call that gave up on a wait can
    // leave them raised); the partials are written before they are read
    if (cudaMemsetAsync(dc.ticket, 0, (size_t)ticket_bytes, s) != cudaSuccess) return ZHA_ERR_CUDA;
    if (launch_dense(dc, n_cta, s) != cudaSuccess) return ZHA_ERR_CUDA;
    return ZHA_OK;
}

}  // extern "C"
