// Internal declarations shared by the blin host layer and its kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <nvtx3/nvToolsExt.h>

#include <mutex>

#include "../../include/blin.h"

namespace blin {

// A named NVTX range around one library call, so that profiler timelines group
// a call's launches under its entry point.  Without an attached tool the push
// and pop are calls to empty functions.
struct TraceRange {
    explicit TraceRange(const char *name) { nvtxRangePushA(name); }
    ~TraceRange() { nvtxRangePop(); }
    TraceRange(const TraceRange &) = delete;
    TraceRange &operator=(const TraceRange &) = delete;
};

// Tokens per TMA tile (and MMA row block).
constexpr int kTile = 128;
// CUDA-core path: state chunks of 1024 tokens counted from the start of their
// block (a function of the block alone, so streamed calls reduce like prefill).
constexpr int kChunk = 1024;

// Element strides of one [B][H][N][d] operand (d innermost, stride 1).
struct Layout {
    long long tok, head, batch;
};

// Geometry of one call, shared by all kernels of that call.
struct KGeom {
    int BH;               // B * H
    int H;                // heads per batch entry
    int N;                // tokens per head in this call
    int T, Hg, Wg, HW;    // latent grid of the call
    int t0;               // absolute index of the call's first frame
    int F;                // frames per full block
    int first_end;        // relative frame at which block 0 ends
    int nblk;             // blocks touched by the call
    int cpb;              // state chunks per block, most of any block (stride of the partial buffer)
    int pt, py, px;       // RoPE pairs per axis (t, y, x)
    float eps;
    const float2 *tab;    // (cos, sin): [T][pt] then [Hg][py] then [Wg][px] (CUDA-core path)
    int tab_y, tab_x;     // offsets (in float2) of the y and x tables
    float *part;          // [BH][nblk][cpb][d*d + d] chunk partial states
    float *prefix;        // [BH][nblk][d*d + d] inclusive prefix states S_<=b, z_<=b
    double theta;         // RoPE base
    int tab_smem;         // 1: the RoPE table fits the tensor-core kernel's shared memory
    int tab_smem_bytes;   // bytes of the whole table (t, y and x parts)
    const float *S_in, *z_in;  // cache entering the call (NULL: zero)
    float *S_out, *z_out;      // cache after the call (NULL: not written)
    Layout lq, lo;             // element strides of q, k, v (shared) and of o
    int swap_q;                // 1: the q/k/v tensor maps order the head dimension before the token one
    // NVFP4 inputs: scale bytes [B*H*N][d/16] of q, k, v and the tensors' global scales
    const uint8_t *sq_scale, *sk_scale, *sv_scale;
    float gq, gk, gv;
    // ---- work units: every block is split into state chunks (pass 1) and, on the
    // tensor-core path, query groups (pass 2) of whole tiles; the first, middle and
    // last blocks of a call may differ in length.
    int nc_first, nc_mid, nc_last;  // state chunks of the first, a middle and the last block
    int ng_first, ng_mid, ng_last;  // query groups of the same
    int U1, U2;                     // pass-1 / pass-2 units of one head
    unsigned int *ctl;    // [4] work counters of the tensor-core kernels, zeroed before each call
};

// Units of block b (nf, nm, nl: of the first, a middle and the last block).
__host__ __device__ inline int units_of_block(const KGeom &g, int b, int nf, int nm, int nl) {
    return b == 0 ? nf : (b == g.nblk - 1 ? nl : nm);
}

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
    WD_P1_FULL = 1,     // pass-1 transform: K/V tile landing
    WD_P1_EMPTY = 2,    // pass-1 producer: landing slot release
    WD_P1_ACC = 3,      // pass-1 accumulator hand-over
    WD_P1_READY = 4,    // pass-1 operand hand-over
    WD_P1_INFO = 5,     // pass-1 chunk record ring
    WD_P1_DRAIN = 6,    // pass-1 final MMA drain
    WD_P2_FULL = 11,    // pass-2 transform: Q tile landing
    WD_P2_EMPTY = 12,   // pass-2 producer: landing slot release
    WD_P2_MMA = 13,     // pass-2 epilogue: accumulator ready
    WD_P2_READY = 14,   // pass-2 operand hand-over
    WD_P2_ACCE = 15,    // pass-2 accumulator release
    WD_P2_BREADY = 16,  // pass-2 prefix / B operand hand-over
    WD_P2_INFO = 17,    // pass-2 tile record ring
    WD_P2_PREFIX = 18,  // pass-2 producer: a head block's prefix state never became ready
    WD_P2_DRAIN = 19,   // pass-2 final MMA drain
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
// Tensor-core path (bf16, d in {32, 64}, splits with a compiled variant): the
// partial-state and output kernels around the block scan.  The maps view
// q/k/v as 4D [B][H][N][d] with the call's strides.
bool tc_supported(int d, const int split[3]);
int tc_table_smem_limit(int d);
// `fp4`: NVFP4 inputs (packed E2M1 data through the maps, scales and global
// scales through the geometry).
cudaError_t launch_partial_tc(const KGeom &g, int d, bool fp4, const CUtensorMap &mk, const CUtensorMap &mv,
                              cudaStream_t s);
cudaError_t launch_output_tc(const KGeom &g, int d, bool fp4, const CUtensorMap &mq, void *o, cudaStream_t s);

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

// Counts one kernel launch in blin_launch_count().
void note_launch();

}  // namespace blin
