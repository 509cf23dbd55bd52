// zha_internal.cuh -- structures shared by the ZHA kernels and the C ABI layer.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "zha_attr.h"

namespace zha {

constexpr int MAXD = 16;          // deepest tree supported
constexpr int BUILD_THREADS = 256;
constexpr int NB = 1024;          // top-p buckets per round
constexpr int CAND_MAX = 768;     // boundary candidates ranked exactly per head
constexpr int SEG_CAP = 256;      // most CTAs in one KV head's team (grid <= 256 CTAs)
constexpr int HIST_ROUNDS = 3;    // bucket widths 1/32, 1/32768, 1/2^25 of a log-mass unit
constexpr int LOC_CAP = 2048;     // frontier slots one CTA holds in shared memory

// Summary store of every level (pointers for KV head 0; head stride is
// node_cap[l] rows).  g: [node][R][d], b and m: [node][R].
struct Tree {
    int h_kv, h_q, G, d, R, c, D, kv_dtype;  // D: current depth
    int c_log2;                   // log2(c) when c is a power of two, else -1
    int64_t kv_cap;               // rows per KV head in K and V
    int64_t n_tokens;             // tokens present
    int32_t n_level[MAXD];        // nodes per level at n_tokens (index l-1)
    int64_t node_cap[MAXD];       // node rows per KV head (index l-1)
    float *g[MAXD];
    float *b[MAXD];
    float *m[MAXD];
    uint16_t *g16[MAXD];          // router copy of g in bf16 ([node][R][d]; null when the router reads g)
    float *b16[MAXD];             // its plane offsets, m - r.g16/sqrt(d) ([node][R])
    const void *K;
    const void *V;
    const float *ref;             // [h_kv][R][d]
    float scale;                  // 1/sqrt(d)
};

// Decode scratch plus outputs of one zha_decode call.  Routing state is kept
// per level l (index l-1) and KV head in "segment" layout: the CTA of team rank
// r that cut level l writes its kept nodes, ascending, at the start of its own
// slot range [S*r/T, S*(r+1)/T) of the level's frontier (S slots, T ranks);
// seg[] holds how many.  Concatenating the segments in rank order gives the
// kept nodes in ascending id order.
struct Decode {
    Tree t;
    int nvk;                      // virtual KV heads: (query of the batch, KV head) pairs, n_q * h_kv;
                                  // virtual head v routes query v / h_kv against KV head v % h_kv, and
                                  // every scratch array, team and output is indexed by v
    const float *q;               // [n_q][h_q][d] = [nvk][G][d]
    float p;
    int32_t *kept_ids[MAXD];      // [h_kv][slot_cap[l-1]] kept node ids (segments)
    uint8_t *kept_mask[MAXD];     // [h_kv][slot_cap[l-1]] heads that kept the node
    int64_t slot_cap[MAXD];       // frontier slots per KV head at level l
    uint32_t *seg;                // [MAXD][h_kv][SEG_CAP] kept nodes per team rank
    uint32_t *hseg;               // [MAXD][h_kv][SEG_CAP][G] kept nodes per team rank and head
    int32_t *lvl;                 // [MAXD][h_kv][2] team size and frontier size of level l
    float *scores;                // [h_kv][score_cap][G] scores when a rank's slots overflow shared memory
    float *rd_scores;             // [h_kv][2][LOC_CAP][G] slices of LV_SPLIT levels (two buffers in turn)
    int32_t *slot_node;           // [h_kv][score_cap] node of each slot (same case)
    uint8_t *slot_keep;           // [h_kv][score_cap] kept heads of each slot (same case)
    int64_t score_cap;
    float *tmax;                  // [h_kv][SEG_CAP][G] per-rank maximum estimate
    uint32_t *tcnt;               // [h_kv][SEG_CAP][G] per-rank frontier count
    unsigned long long *tsum;     // [h_kv][SEG_CAP][G] per-rank boundary mass (slot-order cut)
    uint32_t *hist_cnt;           // [h_kv][HIST_ROUNDS][G][NB]
    unsigned long long *hist_mass;  // [h_kv][HIST_ROUNDS][G][NB]
    unsigned long long *cand_w;   // [h_kv][G][CAND_MAX]
    uint32_t *cand_slot;          // [h_kv][G][CAND_MAX]
    uint32_t *cand_cnt;           // [h_kv][G]
    uint32_t *ticket;             // [h_kv] merge tickets of the attention partials
    float *part;                  // attention partials [part_cap][h_kv][G][d+4]
    int part_cap;
    unsigned *sync;               // barrier words, see zha_sync.cuh
    int64_t *phase_ns;            // nullable: globaltimer stamps per decode phase
    long long wait_budget;        // clock cycles one inter-CTA barrier wait may take
    int32_t *status;
    float *out;
    int32_t *leaf_idx;
    int32_t leaf_cap;
    int32_t *n_leaf;
    int64_t *visited;
    int32_t *trace_ids;
    int32_t *trace_cnt;
    int32_t trace_cap;
};

// device status codes (the values of include/zha.h)
constexpr int32_t ZHA_CAPACITY_CODE = -2;
constexpr int32_t ZHA_TIMEOUT_CODE = -5;

// status word helpers (first error wins)
__device__ __forceinline__ void set_status(int32_t *status, int32_t code) {
    atomicCAS(status, 0, code);
}

// Let kernel `fn` use `bytes` of dynamic shared memory on the current device.
// The attribute is per device: `rec` (one static record per kernel) makes
// the call once per device and size.
template <typename Fn>
cudaError_t allow_smem(Fn *fn, size_t bytes, PerDeviceMax<> &rec) {
    int dev = 0;
    const cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    return static_cast<cudaError_t>(rec.raise(dev, (long long)bytes, [&](long long b) {
        return static_cast<int>(cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)b));
    }));
}

// host-side launchers; each returns a cudaError_t (0 on success)
cudaError_t launch_build(const Tree &t, cudaStream_t s, int n_sm);
cudaError_t launch_append(const Tree &t, const void *k, const void *v, cudaStream_t s);
cudaError_t launch_build_levels(const Tree &t, int from, int to, cudaStream_t s, int n_sm);
cudaError_t launch_decode(const Decode &dc, int n_cta, cudaStream_t s);
int decode_blocks_per_sm(const Decode &dc);
cudaError_t launch_dense(const Decode &dc, int n_cta, cudaStream_t s);
bool compiled_combo(int kv_dtype, int d, int R, int G, int router);

}  // namespace zha
