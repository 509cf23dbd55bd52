// zha_internal.cuh -- structures shared by the ZHA kernels and the C ABI layer.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace zha {

constexpr int MAXD = 16;          // deepest tree supported
constexpr int ROUTE_THREADS = 256;
constexpr int ATTN_THREADS = 256;
constexpr int BUILD_THREADS = 256;
constexpr int NB = 1024;          // coarse top-p buckets per frontier
constexpr float BUCKETS_PER_UNIT = 32.f;  // bucket width 1/32 of a log-mass unit
constexpr int CAND_MAX = 256;     // boundary candidates ranked exactly
constexpr int STAGE_BYTES = 128 * 1024;   // frontier scores staged in shared memory

// Summary store of every level (pointers for KV head 0; head stride is
// node_cap[l] rows).  g: [node][R][d], b and m: [node][R].
struct Tree {
    int h_kv, h_q, G, d, R, c, D, kv_dtype;
    int c_log2;                   // log2(c) when c is a power of two, else -1
    int64_t kv_cap;               // rows per KV head in K and V
    int64_t n_tokens;             // tokens present
    int32_t n_level[MAXD];        // nodes per level at n_tokens (index l-1)
    int64_t node_cap[MAXD];       // node rows per KV head (index l-1)
    float *g[MAXD];
    float *b[MAXD];
    float *m[MAXD];
    const void *K;
    const void *V;
    const float *ref;             // [h_kv][R][d]
    float scale;                  // 1/sqrt(d)
};

// Decode scratch plus outputs of one zha_decode call.
struct Decode {
    Tree t;
    const float *q;               // [h_q][d]
    float p;
    int32_t *kept_ids[MAXD];      // level l: [h_kv][node_cap[l-1]] ascending union kept ids
    uint8_t *kept_mask[MAXD];     // head bitmask per kept id
    int32_t *kept_cnt;            // [MAXD][h_kv]
    float *scores;                // [h_kv][score_cap][G]; -inf where the head does not need the slot
    int32_t *slot_node;           // [h_kv][score_cap] node id of each frontier slot
    int64_t score_cap;
    float *pmax;                  // [h_kv][pmax_cap][G]
    int pmax_cap;
    uint32_t *done;               // [MAXD][h_kv] level tickets, then [h_kv] attention tickets
    int64_t *vis_acc;             // [h_q]
    float *part;                  // attention partials [part_cap][h_kv][G][d+4]
    int part_cap;
    unsigned *gbar;               // grid barrier: arrivals, generation, abort flag
    int64_t *phase_ns;            // nullable: globaltimer stamps per decode phase
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

// host-side launchers; each returns a cudaError_t (0 on success)
cudaError_t launch_build(const Tree &t, cudaStream_t s, int n_sm);
cudaError_t launch_append(const Tree &t, const void *k, const void *v, cudaStream_t s);
cudaError_t launch_decode(const Decode &dc, int n_cta, cudaStream_t s);
int decode_blocks_per_sm(const Decode &dc);
cudaError_t launch_dense(const Decode &dc, int n_cta, cudaStream_t s);
bool compiled_combo(int kv_dtype, int d, int R, int G);

}  // namespace zha
