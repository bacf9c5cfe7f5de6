// Internal declarations shared by the blin host layer and its kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/blin.h"

namespace blin {

// Tokens per TMA tile (and MMA row block) and tiles per state chunk.
constexpr int kTile = 128;
constexpr int kChunkTiles = 8;
constexpr int kChunk = kTile * kChunkTiles;  // 1024 tokens: fixed per block => bit-exact streaming
constexpr int kQTiles = 8;                    // most query tiles per output group

// Geometry of one call, shared by all kernels of that call.
struct KGeom {
    int BH;               // B * H
    int N;                // tokens per head in this call
    int T, Hg, Wg, HW;    // latent grid of the call
    int t0;               // absolute index of the call's first frame
    int F;                // frames per full block
    int first_end;        // relative frame at which block 0 ends
    int nblk;             // blocks touched by the call
    int cpb;              // state chunks per block (stride of the partial buffer)
    int qcpb;             // output groups per block
    int qgt;              // query tiles per output group (<= kQTiles; fewer when a call has few tiles)
    int pt, py, px;       // RoPE pairs per axis (t, y, x)
    float eps;
    const float2 *tab;    // (cos, sin): [T][pt] then [Hg][py] then [Wg][px]
    int tab_y, tab_x;     // offsets (in float2) of the y and x tables
    float *part;          // [BH][nblk][cpb][d*d + d] chunk partial states
    float *prefix;        // [BH][nblk][d*d + d] inclusive prefix states S_<=b, z_<=b
    unsigned int *sched;  // [4] work counters for dynamic scheduling, zeroed before each call
    int chunks_per_bh;    // state chunks of one head in this call
    double theta;         // RoPE base
    int tab_smem;         // 1: the RoPE table fits the tensor-core kernels' shared memory
    int tab_smem_bytes;   // bytes of the whole table (t, y and x parts)
    const float *S_in, *z_in;  // cache entering the call (NULL: zero)
    float *S_out, *z_out;      // cache after the call (NULL: not written)
};

__host__ __device__ inline int block_frame_begin(const KGeom &g, int b) {
    return b == 0 ? 0 : g.first_end + (b - 1) * g.F;
}
__host__ __device__ inline int block_frame_end(const KGeom &g, int b) {
    int e = g.first_end + b * g.F;
    return e < g.T ? e : g.T;
}

// Device-side watchdog word: 0 = fine, otherwise the code of the wait that ran out.
enum WatchdogCode : int {
    WD_NONE = 0,
    WD_PARTIAL_FULL = 1,
    WD_PARTIAL_EMPTY = 2,
    WD_PARTIAL_ACC = 3,
    WD_PARTIAL_READY = 4,
    WD_OUT_FULL = 11,
    WD_OUT_EMPTY = 12,
    WD_OUT_MMA = 13,
    WD_OUT_READY = 14,
    WD_OUT_ACCE = 15,
    WD_OUT_BREADY = 16,
};

// Launchers (all enqueue on `s`; return the launch's cudaError_t).
// Fills the RoPE table in global memory (CUDA-core path).
cudaError_t launch_rope_table(const KGeom &g, cudaStream_t s);
cudaError_t launch_scan(const KGeom &g, int d, const float *S_in, const float *z_in, float *S_out,
                        float *z_out, cudaStream_t s);
cudaError_t launch_partial_simt(const KGeom &g, int d, bool bf16, const void *k, const void *v,
                                cudaStream_t s);
cudaError_t launch_output_simt(const KGeom &g, int d, bool bf16, const void *q, void *o,
                               cudaStream_t s);
// Tensor-core path (bf16, d in {32, 64}, splits with a compiled variant).
bool tc_supported(int d, const int split[3]);
// Chunk partial states (the block scan follows as its own launch).
cudaError_t launch_partial_tc(const KGeom &g, int d, const CUtensorMap &mk, const CUtensorMap &mv,
                              cudaStream_t s);
// Shared-memory bytes the tensor-core kernels need for a RoPE table copy of
// `entries` float2 (0 when the table is read from global memory).
int tc_table_smem_limit(int d);
cudaError_t launch_output_tc(const KGeom &g, int d, const CUtensorMap &mq, const CUtensorMap &mo, void *o,
                             cudaStream_t s);

// Device watchdog access.
cudaError_t read_and_clear_watchdog(int *code);

// Unique id of the calling thread's current CUDA context (0 if none or the
// driver cannot tell).  Device addresses and function attributes belong to a
// context, so per-context caches key on this, not on the device ordinal: a
// host framework may make another context current, and cudaDeviceReset
// replaces the primary one.
unsigned long long current_context_id();

// A small cache of per-context values (device addresses, flags), keyed by
// current_context_id(); thread safe.
template <typename V>
struct ContextCache {
    static constexpr int kSlots = 32;
    std::mutex mu;
    unsigned long long key[kSlots] = {};
    V val[kSlots] = {};
    int next = 0;
    bool get(unsigned long long k, V *out) {
        std::lock_guard<std::mutex> lock(mu);
        for (int i = 0; i < kSlots; ++i)
            if (key[i] == k && k != 0) {
                *out = val[i];
                return true;
            }
        return false;
    }
    void put(unsigned long long k, V v) {
        if (k == 0) return;
        std::lock_guard<std::mutex> lock(mu);
        for (int i = 0; i < kSlots; ++i)
            if (key[i] == k) {
                val[i] = v;
                return;
            }
        key[next] = k;
        val[next] = v;
        next = (next + 1) % kSlots;
    }
};

// Records `msg` as this thread's blin_last_error() text and returns `st`.
blin_status set_last_error(blin_status st, const char *msg);

}  // namespace blin
