// Host side of libblin: argument checks, the (S, z) state object, workspace
// layout, TMA descriptors and the launch sequence of each call.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <atomic>
#include <mutex>

#include "../../include/blin.h"
#include "blin_internal.cuh"

using namespace blin;

static constexpr uint64_t kStateMagic = 0x626c696e53544154ull;  // "blinSTAT"
static constexpr uint64_t kFreedMagic = 0xdeadbeefdeadbeefull;

struct blin_state {
    uint64_t magic;
    int B, H, d, device;
    float *S;  // [B][H][d][d]
    float *z;  // [B][H][d]
    int t_next;
    void *scratch;  // block-step workspace (tables, partials, prefix)
    size_t scratch_bytes;
    cudaEvent_t last_use;  // recorded after every call that reads or writes S, z or the scratch
};

static thread_local char g_err[512] = "";
static thread_local int g_last_path = 0;  // blin_path of this thread's last call that launched kernels

static blin_status fail(blin_status st, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return st;
}

blin_status blin::set_last_error(blin_status st, const char *msg) { return fail(st, "%s", msg); }

static blin_status cuda_fail(cudaError_t e, const char *what) {
    return fail(BLIN_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// ---------------------------------------------------------------- geometry
struct Plan {
    KGeom g;
    int d;
    bool tc;  // tensor-core path
    size_t ctl_bytes, tab_bytes, part_bytes, prefix_bytes;
};

static blin_status check_common(int B, int H, int d, int T, int Hg, int Wg, const int split[3],
                                float theta, float eps) {
    if (B < 1 || H < 1) return fail(BLIN_ERR_INVALID_ARG, "B and H must be >= 1 (got %d, %d)", B, H);
    if (d != 32 && d != 64) return fail(BLIN_ERR_SHAPE, "head dim d must be 32 or 64 (got %d)", d);
    if (T < 0) return fail(BLIN_ERR_INVALID_ARG, "T must be >= 0 (got %d)", T);
    if (Hg < 1 || Wg < 1) return fail(BLIN_ERR_INVALID_ARG, "Hgt and Wid must be >= 1 (got %d, %d)", Hg, Wg);
    if (split == nullptr) return fail(BLIN_ERR_INVALID_ARG, "rope_split is NULL");
    for (int a = 0; a < 3; ++a)
        if (split[a] < 0 || (split[a] & 1))
            return fail(BLIN_ERR_SHAPE, "rope_split entries must be even and >= 0 (got %d,%d,%d)",
                        split[0], split[1], split[2]);
    if (split[0] + split[1] + split[2] != d)
        return fail(BLIN_ERR_SHAPE, "rope_split (%d,%d,%d) must sum to d=%d", split[0], split[1], split[2], d);
    if (!(theta > 0.f) || !std::isfinite(theta)) return fail(BLIN_ERR_INVALID_ARG, "theta must be finite and > 0");
    if (!(eps >= 0.f) || !std::isfinite(eps)) return fail(BLIN_ERR_INVALID_ARG, "eps must be finite and >= 0");
    const long long HW = (long long)Hg * Wg;
    const long long N = (long long)T * HW;
    const long long rows = (long long)B * H * N;
    if (HW > (1 << 30) || N >= (1LL << 31) || rows >= (1LL << 40) || (long long)B * H >= (1LL << 24))
        return fail(BLIN_ERR_SHAPE, "problem too large (B*H*N = %lld rows)", rows);
    return BLIN_OK;
}

// Tensor-core path, pass 1: state chunks per block, of about kChunkTiles32 /
// kChunkTiles64 tiles, split evenly.  The count is a function of the block's
// length and d only (never of the call, the number of heads or the device), so
// a head's block reduces in the same chunks whether it arrives in a prefill, in
// a block step or in a call with other heads.
static constexpr int kChunkTiles32 = 5, kChunkTiles64 = 8;
static int tc_chunks(long long L, int d) {
    const long long nt = (L + kTile - 1) / kTile;
    const long long ct = d == 32 ? kChunkTiles32 : kChunkTiles64;
    return (int)std::max(1LL, (nt + ct - 1) / ct);
}
// Tensor-core path, pass 2: query groups of up to `gt` tiles per block (the
// grouping does not change any output bit).
static int tc_groups(long long L, int gt) {
    const long long nt = (L + kTile - 1) / kTile;
    return (int)std::max(1LL, (nt + gt - 1) / gt);
}
// CUDA-core path: 1024-token chunks.
static int simt_chunks(long long L) { return (int)std::max(1LL, (L + kChunk - 1) / kChunk); }

// Builds the call geometry; `one_block` treats the whole call as one block;
// `for_size` sizes for the worst case over the starting frame (and both paths).
static Plan make_plan(int B, int H, int d, int T, int Hg, int Wg, int F, int t0, bool one_block,
                      const int split[3], float eps, bool tc, bool for_size = false) {
    Plan p{};
    KGeom &g = p.g;
    p.d = d;
    g.BH = B * H;
    g.H = H;
    g.T = T;
    g.Hg = Hg;
    g.Wg = Wg;
    g.HW = Hg * Wg;
    g.N = T * g.HW;
    g.t0 = t0;
    if (one_block) {
        g.F = T > 0 ? T : 1;
        g.first_end = T;
        g.nblk = T > 0 ? 1 : 0;
    } else {
        g.F = F;
        const int fe = (t0 / F + 1) * F - t0;  // relative frame where the first block ends
        g.first_end = fe < T ? fe : T;
        g.nblk = T > 0 ? 1 + (T - g.first_end + F - 1) / F : 0;
        if (for_size) g.nblk = (T + F - 1) / F + 1;  // worst case over t0
    }
    g.pt = split[0] / 2;
    g.py = split[1] / 2;
    g.px = split[2] / 2;
    g.eps = eps;
    g.tab_y = T * g.pt;
    g.tab_x = g.tab_y + Hg * g.py;
    // The tensor-core kernel keeps the call's whole RoPE table in shared memory;
    // a call whose table does not fit next to its rings takes the CUDA-core path.
    const long long tab_entries = (long long)T * g.pt + (long long)Hg * g.py + (long long)Wg * g.px;
    g.tab_smem_bytes = (int)std::min<long long>(tab_entries * (long long)sizeof(float2), 1 << 30);
    g.tab_smem = g.tab_smem_bytes <= tc_table_smem_limit(d) ? 1 : 0;
    tc = tc && g.tab_smem;
    p.tc = tc;
    // block lengths (tokens): the first, a middle and the last block
    const long long HW = g.HW;
    const long long Lf = (long long)g.first_end * HW, Lm = (long long)g.F * HW;
    const long long Ll = g.nblk >= 2 ? (long long)(T - g.first_end - (g.nblk - 2) * g.F) * HW : Lf;
    const long long Lmax = (long long)(one_block ? T : std::min(F, T)) * HW;
    const int mids = g.nblk > 2 ? g.nblk - 2 : 0;
    if (for_size) {
        g.cpb = std::max(tc_chunks(Lmax, d), simt_chunks(Lmax));
    } else {
        auto chunks = [&](long long L) { return tc ? tc_chunks(L, d) : simt_chunks(L); };
        g.nc_first = chunks(Lf);
        g.nc_mid = chunks(Lm);
        g.nc_last = chunks(Ll);
        // query groups of 8 tiles (the B operand is rebuilt once per group), fewer when
        // the call has too few groups to keep every pass-2 pipeline of a B200 busy
        int gt = 8;
        auto all_groups = [&](int t) {
            return (long long)g.BH * (tc_groups(Lf, t) + (long long)mids * tc_groups(Lm, t) + (g.nblk >= 2 ? tc_groups(Ll, t) : 0));
        };
        while (gt > 2 && all_groups(gt) < 3 * 296) gt /= 2;
        g.ng_first = tc_groups(Lf, gt);
        g.ng_mid = tc_groups(Lm, gt);
        g.ng_last = tc_groups(Ll, gt);
        g.U1 = g.nblk == 0 ? 0 : g.nc_first + mids * g.nc_mid + (g.nblk >= 2 ? g.nc_last : 0);
        g.U2 = g.nblk == 0 ? 0 : g.ng_first + mids * g.ng_mid + (g.nblk >= 2 ? g.ng_last : 0);
        g.cpb = std::max(g.nc_first, g.nblk >= 2 ? g.nc_last : 0);
        if (mids > 0) g.cpb = std::max(g.cpb, g.nc_mid);
    }
    if (g.cpb < 1) g.cpb = 1;
    const size_t E = (size_t)d * d + d;
    p.ctl_bytes = 256;  // work counters
    p.tab_bytes = align256(sizeof(float2) * ((size_t)T * g.pt + (size_t)Hg * g.py + (size_t)Wg * g.px + 1));
    p.part_bytes = align256(sizeof(float) * (size_t)g.BH * g.nblk * g.cpb * E);
    p.prefix_bytes = align256(sizeof(float) * (size_t)g.BH * g.nblk * E);
    // contiguous [B][H][N][d] unless the caller says otherwise
    g.lq = g.lo = Layout{d, (long long)g.N * d, (long long)H * g.N * d};
    return p;
}

// Launch-shape limits of a plan.  The tensor-core kernels hand out the call's
// (head, chunk) and (head, query group) units through 32-bit counters that run a
// few claims past the end; the CUDA-core kernels put blocks and heads on grid y
// and z, which hold at most 65535 each.
static constexpr long long kMaxUnits = (1LL << 31) - (1LL << 20);
static blin_status check_launch_limits(const Plan &p) {
    const KGeom &g = p.g;
    if (p.tc) {
        const long long u1 = (long long)g.BH * g.U1, u2 = (long long)g.BH * g.U2;
        if (u1 > kMaxUnits || u2 > kMaxUnits)
            return fail(BLIN_ERR_SHAPE, "too many work units for one call (%lld state chunks, %lld query groups); "
                                        "split the call over heads or frames", u1, u2);
    } else if (g.BH > 65535 || g.nblk > 65535) {
        return fail(BLIN_ERR_SHAPE, "the CUDA-core path takes at most 65535 heads (B*H = %d) and 65535 blocks "
                                    "(%d) per call; split the call", g.BH, g.nblk);
    }
    return BLIN_OK;
}

// 256 bytes of alignment slack, then the work counters, RoPE table, chunk partials, prefixes
static size_t plan_bytes(const Plan &p) { return 256 + p.ctl_bytes + p.tab_bytes + p.part_bytes + p.prefix_bytes; }

static void plan_bind(Plan &p, void *ws) {
    uintptr_t base = (reinterpret_cast<uintptr_t>(ws) + 255) & ~uintptr_t(255);
    p.g.ctl = reinterpret_cast<unsigned int *>(base);
    base += p.ctl_bytes;
    p.g.tab = reinterpret_cast<const float2 *>(base);
    p.g.part = reinterpret_cast<float *>(base + p.tab_bytes);
    p.g.prefix = reinterpret_cast<float *>(base + p.tab_bytes + p.part_bytes);
}

// Bytes of a prefill workspace for this shape (both paths, any starting frame).
static size_t prefill_bytes(int B, int H, int d, const blin_geom *g) {
    Plan p = make_plan(B, H, d, g->T, g->Hgt, g->Wid, g->block_frames, 0, false, g->rope_split, g->eps, false, true);
    return plan_bytes(p);
}

// ---------------------------------------------------------------- contexts
typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

unsigned long long blin::current_context_id() {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(p);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(p);
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_current == nullptr || get_id == nullptr || get_current(&ctx) != CUDA_SUCCESS) return 0;
    if (ctx == nullptr) {  // no context yet: let the runtime bind the device's primary one
        cudaFree(nullptr);
        if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
    }
    if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// ---------------------------------------------------------------- TMA descriptors
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// 4D view of a bf16 [B][H][N][d] operand with element strides `l`: dimensions
// (feature, then token and head ordered by stride, then batch), `box_rows`
// tokens per box, swizzled to the row size (64 B at d = 32, 128 B at d = 64).
// *swap = 1 when the head dimension comes before the token one.  Tokens past
// N read as zeros.
static bool make_map4(CUtensorMap *m, const void *base, const Layout &l, int B, int H, int N, int d, int box_rows,
                      int *swap) {
    EncodeTiledFn enc = encode_fn();
    if (enc == nullptr) return false;
    const bool sw = l.head < l.tok;
    *swap = sw ? 1 : 0;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)(sw ? H : N), (cuuint64_t)(sw ? N : H), (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)(sw ? l.head : l.tok) * 2, (cuuint64_t)(sw ? l.tok : l.head) * 2,
                             (cuuint64_t)l.batch * 2};
    cuuint32_t box[4] = {(cuuint32_t)d, (cuuint32_t)(sw ? 1 : box_rows), (cuuint32_t)(sw ? box_rows : 1), 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, d == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 4D view of NVFP4 packed data [B][H][N][d/2] bytes (contiguous): `box_rows`
// tokens per box, no swizzle.  Tokens past N read as zeros.
static bool make_map4_fp4(CUtensorMap *m, const void *base, int B, int H, int N, int d, int box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (enc == nullptr) return false;
    const cuuint64_t rowb = (cuuint64_t)d / 2;
    cuuint64_t dims[4] = {rowb, (cuuint64_t)N, (cuuint64_t)H, (cuuint64_t)B};
    cuuint64_t strides[3] = {rowb, rowb * N, rowb * N * H};
    cuuint32_t box[4] = {(cuuint32_t)rowb, (cuuint32_t)box_rows, 1, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void *>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// NVFP4 operands of one call (NULL: bf16 / fp32 operands).
struct Fp4In {
    const blin_nvfp4 *q, *k, *v;
};

// ---------------------------------------------------------------- launch sequence
static thread_local cudaEvent_t const *g_timing = nullptr;

// Kernels this library has launched in this process (all threads, all devices).
static std::atomic<unsigned long long> g_launches{0};

void blin::note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

static void mark(int i, bool after, cudaStream_t s) {
    if (g_timing != nullptr) cudaEventRecord(g_timing[2 * i + (after ? 1 : 0)], s);
}

// Enqueues the call.
static blin_status run(Plan &p, const void *q, const void *k, const void *v, void *o, blin_dtype dt,
                       const float *S_in, const float *z_in, float *S_out, float *z_out, double theta,
                       cudaStream_t s, const Fp4In *fp4 = nullptr) {
    p.g.S_in = S_in;
    p.g.z_in = z_in;
    p.g.theta = theta;
    p.g.S_out = S_out;
    p.g.z_out = z_out;
    KGeom &g = p.g;
    const int d = p.d;
    const bool tc = p.tc;
    g_last_path = tc ? BLIN_PATH_TENSOR_CORE : BLIN_PATH_CUDA_CORE;
    cudaError_t e;
    if (tc) {
        CUtensorMap mq, mk, mv;
        int sk = 0, sv = 0;
        const int B = g.BH / g.H;
        bool maps;
        if (fp4) {
            g.swap_q = 0;
            g.sq_scale = static_cast<const uint8_t *>(fp4->q->scale);
            g.sk_scale = static_cast<const uint8_t *>(fp4->k->scale);
            g.sv_scale = static_cast<const uint8_t *>(fp4->v->scale);
            g.gq = fp4->q->global_scale;
            g.gk = fp4->k->global_scale;
            g.gv = fp4->v->global_scale;
            maps = make_map4_fp4(&mq, q, B, g.H, g.N, d, kTile) && make_map4_fp4(&mk, k, B, g.H, g.N, d, kTile) &&
                   make_map4_fp4(&mv, v, B, g.H, g.N, d, kTile);
        } else {
            maps = make_map4(&mq, q, g.lq, B, g.H, g.N, d, kTile, &g.swap_q) &&
                   make_map4(&mk, k, g.lq, B, g.H, g.N, d, kTile, &sk) && make_map4(&mv, v, g.lq, B, g.H, g.N, d, kTile, &sv);
        }
        if (!maps)
            return fail(BLIN_ERR_CUDA, "cuTensorMapEncodeTiled failed (driver entry point unavailable or strides rejected)");
        // both kernels hand out their work through counters that start at zero
        if ((e = cudaMemsetAsync(g.ctl, 0, 4 * sizeof(unsigned int), s)) != cudaSuccess)
            return cuda_fail(e, "work counter reset");
        mark(1, false, s);
        if ((e = launch_partial_tc(g, d, fp4 != nullptr, mk, mv, s)) != cudaSuccess)
            return cuda_fail(e, "partial-state launch");
        g_launches.fetch_add(1, std::memory_order_relaxed);
        mark(1, true, s);
        mark(2, false, s);
        if ((e = launch_scan(g, d, S_in, z_in, S_out, z_out, s)) != cudaSuccess) return cuda_fail(e, "scan launch");
        g_launches.fetch_add(1, std::memory_order_relaxed);
        mark(2, true, s);
        mark(3, false, s);
        if ((e = launch_output_tc(g, d, fp4 != nullptr, mq, o, s)) != cudaSuccess) return cuda_fail(e, "output launch");
        g_launches.fetch_add(1, std::memory_order_relaxed);
        mark(3, true, s);
        return BLIN_OK;
    }
    const bool bf = dt == BLIN_BF16;
    mark(0, false, s);
    if ((e = launch_rope_table(g, s)) != cudaSuccess) return cuda_fail(e, "rope table launch");
    g_launches.fetch_add(1, std::memory_order_relaxed);
    mark(0, true, s);
    mark(1, false, s);
    if ((e = launch_partial_simt(g, d, bf, k, v, s)) != cudaSuccess) return cuda_fail(e, "partial-state launch");
    g_launches.fetch_add(1, std::memory_order_relaxed);
    mark(1, true, s);
    mark(2, false, s);
    if ((e = launch_scan(g, d, S_in, z_in, S_out, z_out, s)) != cudaSuccess) return cuda_fail(e, "scan launch");
    g_launches.fetch_add(1, std::memory_order_relaxed);
    mark(2, true, s);
    mark(3, false, s);
    if ((e = launch_output_simt(g, d, bf, q, o, s)) != cudaSuccess) return cuda_fail(e, "output launch");
    g_launches.fetch_add(1, std::memory_order_relaxed);
    mark(3, true, s);
    return BLIN_OK;
}

// Records the state's last-use event on `s` (blin_state_free waits for it).
// Work captured into a CUDA graph is not marked: it runs when the graph is
// launched, which the library does not see.
static blin_status mark_state_use(blin_state *st, cudaStream_t s) {
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    cudaError_t e = cudaStreamIsCapturing(s, &cap);
    if (e != cudaSuccess) return cuda_fail(e, "stream capture query");
    if (cap != cudaStreamCaptureStatusNone) return BLIN_OK;
    e = cudaEventRecord(st->last_use, s);
    return e == cudaSuccess ? BLIN_OK : cuda_fail(e, "state event record");
}

static blin_status check_state(const blin_state *st) {
    if (st == nullptr) return fail(BLIN_ERR_INVALID_ARG, "state is NULL");
    if (st->magic != kStateMagic) return fail(BLIN_ERR_STATE, "state handle is not live (freed or foreign)");
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != st->device)
        return fail(BLIN_ERR_STATE, "state lives on device %d but the current device is %d", st->device, dev);
    return BLIN_OK;
}

static blin_status check_io(const void *q, const void *k, const void *v, void *o, blin_dtype dt) {
    if (q == nullptr || k == nullptr || v == nullptr || o == nullptr)
        return fail(BLIN_ERR_INVALID_ARG, "q, k, v and o must be non-NULL device pointers");
    if (dt != BLIN_F32 && dt != BLIN_BF16) return fail(BLIN_ERR_DTYPE, "unknown dtype %d", (int)dt);
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
        return fail(BLIN_ERR_ALIGN, "q, k, v and o must be 16-byte aligned");
    return BLIN_OK;
}

extern "C" {

const char *blin_last_error(void) { return g_err; }

const char *blin_version(void) { return "blin 0.1 (sm_100a)"; }

blin_status blin_state_init(int B, int H, int d, blin_stream stream, blin_state **out) {
    if (out == nullptr) return fail(BLIN_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    if (B < 1 || H < 1) return fail(BLIN_ERR_INVALID_ARG, "B and H must be >= 1");
    if (d != 32 && d != 64) return fail(BLIN_ERR_SHAPE, "d must be 32 or 64");
    blin_state *st = new blin_state{};
    st->magic = kStateMagic;
    st->B = B;
    st->H = H;
    st->d = d;
    cudaError_t e = cudaGetDevice(&st->device);
    const size_t sb = sizeof(float) * (size_t)B * H * d * d, zb = sizeof(float) * (size_t)B * H * d;
    if (e == cudaSuccess) e = cudaMalloc(&st->S, sb);
    if (e == cudaSuccess) e = cudaMalloc(&st->z, zb);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(st->S, 0, sb, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(st->z, 0, zb, s);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&st->last_use, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventRecord(st->last_use, s);
    if (e != cudaSuccess) {
        if (st->S) cudaFree(st->S);
        if (st->z) cudaFree(st->z);
        if (st->last_use) cudaEventDestroy(st->last_use);
        delete st;
        return cuda_fail(e, "state allocation");
    }
    *out = st;
    return BLIN_OK;
}

blin_status blin_state_free(blin_state *st) {
    if (st == nullptr) return BLIN_OK;
    if (st->magic != kStateMagic) return fail(BLIN_ERR_STATE, "state handle is not live (double free?)");
    int prev = 0;
    cudaGetDevice(&prev);
    cudaSetDevice(st->device);
    // wait only for the work that used this state (its last call's stream position)
    cudaError_t e = cudaEventSynchronize(st->last_use);
    cudaEventDestroy(st->last_use);
    cudaFree(st->S);
    cudaFree(st->z);
    if (st->scratch) cudaFree(st->scratch);
    cudaSetDevice(prev);
    st->magic = kFreedMagic;
    delete st;
    if (e != cudaSuccess) return cuda_fail(e, "wait for the state's last use before freeing it");
    return BLIN_OK;
}

blin_status blin_state_reset(blin_state *st, blin_stream stream) {
    blin_status rc = check_state(st);
    if (rc != BLIN_OK) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t sb = sizeof(float) * (size_t)st->B * st->H * st->d * st->d;
    const size_t zb = sizeof(float) * (size_t)st->B * st->H * st->d;
    cudaError_t e = cudaMemsetAsync(st->S, 0, sb, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(st->z, 0, zb, s);
    if (e != cudaSuccess) return cuda_fail(e, "state reset");
    if ((rc = mark_state_use(st, s)) != BLIN_OK) return rc;
    st->t_next = 0;
    return BLIN_OK;
}

blin_status blin_state_tensors(const blin_state *st, float **S, float **z, int *t_next) {
    if (st == nullptr) return fail(BLIN_ERR_INVALID_ARG, "state is NULL");
    if (st->magic != kStateMagic) return fail(BLIN_ERR_STATE, "state handle is not live");
    if (S) *S = st->S;
    if (z) *z = st->z;
    if (t_next) *t_next = st->t_next;
    return BLIN_OK;
}

size_t blin_state_bytes(const blin_state *st) {
    if (st == nullptr || st->magic != kStateMagic) return 0;
    return sizeof(float) * (size_t)st->B * st->H * ((size_t)st->d * st->d + st->d);
}

blin_status blin_state_copy_to_host(const blin_state *st, void *host, size_t bytes, blin_stream stream) {
    blin_status rc = check_state(st);
    if (rc != BLIN_OK) return rc;
    if (host == nullptr) return fail(BLIN_ERR_INVALID_ARG, "host buffer is NULL");
    if (bytes != blin_state_bytes(st))
        return fail(BLIN_ERR_STATE, "bytes=%zu but the state holds %zu", bytes, blin_state_bytes(st));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t sb = sizeof(float) * (size_t)st->B * st->H * st->d * st->d;
    cudaError_t e = cudaMemcpyAsync(host, st->S, sb, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(static_cast<char *>(host) + sb, st->z, bytes - sb, cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) return cuda_fail(e, "state copy to host");
    return mark_state_use(const_cast<blin_state *>(st), s);
}

blin_status blin_state_copy_from_host(blin_state *st, const void *host, size_t bytes, int t_next,
                                      blin_stream stream) {
    blin_status rc = check_state(st);
    if (rc != BLIN_OK) return rc;
    if (host == nullptr) return fail(BLIN_ERR_INVALID_ARG, "host buffer is NULL");
    if (t_next < 0) return fail(BLIN_ERR_INVALID_ARG, "t_next must be >= 0");
    if (bytes != blin_state_bytes(st))
        return fail(BLIN_ERR_STATE, "bytes=%zu but the state holds %zu", bytes, blin_state_bytes(st));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t sb = sizeof(float) * (size_t)st->B * st->H * st->d * st->d;
    cudaError_t e = cudaMemcpyAsync(st->S, host, sb, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(st->z, static_cast<const char *>(host) + sb, bytes - sb, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e, "state copy from host");
    if ((rc = mark_state_use(st, s)) != BLIN_OK) return rc;
    st->t_next = t_next;
    return BLIN_OK;
}

// Grows the state's block-step scratch to `need` bytes.
static blin_status ensure_scratch(blin_state *st, size_t need, cudaStream_t s) {
    if (st->scratch_bytes >= need) return BLIN_OK;
    // Growing inside stream capture would make the state hold graph-owned memory
    // that later calls outside the graph reuse: refuse, and let the caller reserve.
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    cudaError_t e = cudaStreamIsCapturing(s, &cap);
    if (e != cudaSuccess) return cuda_fail(e, "stream capture query");
    if (cap != cudaStreamCaptureStatusNone)
        return fail(BLIN_ERR_WORKSPACE, "the state's block-step scratch must grow to %zu bytes, which cannot happen "
                                        "during stream capture: call blin_state_reserve before capturing", need);
    void *p = nullptr;
    e = cudaMallocAsync(&p, need, s);
    if (e != cudaSuccess) {
        if (p) cudaFreeAsync(p, s);
        return cuda_fail(e, "block-step scratch allocation");
    }
    if (st->scratch) cudaFreeAsync(st->scratch, s);
    st->scratch = p;
    st->scratch_bytes = need;
    return BLIN_OK;
}

// Element strides of q/k/v (or o) from the caller's layout (NULL: contiguous).
static blin_status get_layout(const blin_layout *l, int B, int H, int N, int d, blin_dtype dt, const char *name,
                              Layout *out) {
    if (l == nullptr) {
        *out = Layout{d, (long long)N * d, (long long)H * N * d};
        return BLIN_OK;
    }
    Layout x{l->token, l->head, l->batch};
    // a dimension of extent 1 never moves: give it a harmless stride
    if (H == 1) x.head = x.tok * (long long)std::max(N, 1);
    if (B == 1) x.batch = std::max(x.tok * (long long)std::max(N, 1), x.head * (long long)H);
    if (x.tok < d || x.head < d || x.batch < d)
        return fail(BLIN_ERR_SHAPE, "%s strides (token %lld, head %lld, batch %lld) must each be >= d = %d", name,
                    l->token, l->head, l->batch, d);
    const long long es = dt == BLIN_BF16 ? 2 : 4;
    if ((x.tok * es) % 16 || (x.head * es) % 16 || (x.batch * es) % 16)
        return fail(BLIN_ERR_ALIGN, "%s strides must be multiples of 16 bytes", name);
    if (x.tok * es >= (1LL << 40) || x.head * es >= (1LL << 40) || x.batch * es >= (1LL << 40))
        return fail(BLIN_ERR_SHAPE, "%s strides too large", name);
    *out = x;
    return BLIN_OK;
}

blin_status blin_state_reserve(blin_state *st, long max_block_tokens, blin_stream stream) {
    blin_status rc = check_state(st);
    if (rc != BLIN_OK) return rc;
    if (max_block_tokens < 1 || max_block_tokens >= (1L << 30))
        return fail(BLIN_ERR_INVALID_ARG, "max_block_tokens out of range");
    // Widest table: all tokens on one axis of one frame (Hgt = 1, Wid = tokens).
    const int split_wide[3] = {0, 0, st->d};
    Plan p = make_plan(st->B, st->H, st->d, 1, 1, (int)max_block_tokens, 1, 0, true, split_wide, 0.f, false, true);
    return ensure_scratch(st, plan_bytes(p), static_cast<cudaStream_t>(stream));
}

size_t blin_prefill_workspace_size(int B, int H, int d, const blin_geom *g) {
    if (g == nullptr) return 0;
    if (check_common(B, H, d, g->T, g->Hgt, g->Wid, g->rope_split, g->theta, g->eps) != BLIN_OK) return 0;
    if (g->block_frames < 1) return 0;
    return prefill_bytes(B, H, d, g);
}

static blin_status prefill_impl(const void *q, const void *k, const void *v, void *o, blin_dtype dt, int B, int H,
                                int d, const blin_geom *g, const blin_layout *lqkv, const blin_layout *lout,
                                blin_state *st, void *workspace, size_t ws_bytes, blin_stream stream,
                                const Fp4In *fp4 = nullptr) {
    const TraceRange trace(fp4 ? "blin_prefill_nvfp4" : (lqkv || lout) ? "blin_prefill_strided" : "blin_prefill");
    if (g == nullptr) return fail(BLIN_ERR_INVALID_ARG, "geom is NULL");
    blin_status rc = check_common(B, H, d, g->T, g->Hgt, g->Wid, g->rope_split, g->theta, g->eps);
    if (rc != BLIN_OK) return rc;
    if (g->block_frames < 1) return fail(BLIN_ERR_INVALID_ARG, "block_frames must be >= 1");
    if ((rc = check_io(q, k, v, o, dt)) != BLIN_OK) return rc;
    const int N = g->T * g->Hgt * g->Wid;
    Layout lq, lo;
    if ((rc = get_layout(lqkv, B, H, N, d, dt, "q/k/v", &lq)) != BLIN_OK) return rc;
    if ((rc = get_layout(lout, B, H, N, d, dt, "o", &lo)) != BLIN_OK) return rc;
    if (st != nullptr) {
        if ((rc = check_state(st)) != BLIN_OK) return rc;
        if (st->B != B || st->H != H || st->d != d)
            return fail(BLIN_ERR_STATE, "state is B=%d H=%d d=%d, call is B=%d H=%d d=%d", st->B, st->H,
                        st->d, B, H, d);
    }
    if (g->T == 0) return BLIN_OK;
    const int t0 = st ? st->t_next : 0;
    if ((long long)t0 + g->T >= (1LL << 30)) return fail(BLIN_ERR_SHAPE, "frame index overflow");
    const bool tc = dt == BLIN_BF16 && tc_supported(d, g->rope_split);
    Plan p = make_plan(B, H, d, g->T, g->Hgt, g->Wid, g->block_frames, t0, false, g->rope_split, g->eps, tc);
    if ((rc = check_launch_limits(p)) != BLIN_OK) return rc;
    if (fp4 && !p.tc)
        return fail(BLIN_ERR_SHAPE, "NVFP4 inputs need the tensor-core path (rope split (8,12,12) at d=32 or "
                                    "(16,24,24) at d=64, and a RoPE table that fits shared memory)");
    // the workspace is checked last: every shape and layout check above needs none
    const size_t need = prefill_bytes(B, H, d, g);
    if (workspace == nullptr || ws_bytes < need)
        return fail(BLIN_ERR_WORKSPACE, "workspace of %zu bytes given, %zu needed", workspace ? ws_bytes : 0, need);
    if (!aligned16(workspace)) return fail(BLIN_ERR_ALIGN, "workspace must be 16-byte aligned");
    p.g.lq = lq;
    p.g.lo = lo;
    plan_bind(p, workspace);
    rc = run(p, q, k, v, o, dt, st ? st->S : nullptr, st ? st->z : nullptr, st ? st->S : nullptr,
             st ? st->z : nullptr, (double)g->theta, static_cast<cudaStream_t>(stream), fp4);
    if (rc != BLIN_OK) return rc;
    if (st) {
        if ((rc = mark_state_use(st, static_cast<cudaStream_t>(stream))) != BLIN_OK) return rc;
        st->t_next += g->T;
    }
    return BLIN_OK;
}

static blin_status block_step_impl(const void *q, const void *k, const void *v, void *o, blin_dtype dt, int B,
                                   int H, int d, const blin_geom *g, const blin_layout *lqkv,
                                   const blin_layout *lout, blin_state *st, int commit, blin_stream stream,
                                   const Fp4In *fp4 = nullptr) {
    const TraceRange trace(fp4 ? "blin_block_step_nvfp4"
                               : (lqkv || lout) ? "blin_block_step_strided" : "blin_block_step");
    if (g == nullptr) return fail(BLIN_ERR_INVALID_ARG, "geom is NULL");
    blin_status rc = check_common(B, H, d, g->T, g->Hgt, g->Wid, g->rope_split, g->theta, g->eps);
    if (rc != BLIN_OK) return rc;
    const int frames = g->T, F = g->block_frames;
    if (frames < 1) return fail(BLIN_ERR_INVALID_ARG, "frames (geom T) must be >= 1");
    if (F < 1) return fail(BLIN_ERR_INVALID_ARG, "block_frames must be >= 1");
    if (commit != 0 && commit != 1) return fail(BLIN_ERR_INVALID_ARG, "commit must be 0 or 1");
    if ((rc = check_io(q, k, v, o, dt)) != BLIN_OK) return rc;
    const int N = frames * g->Hgt * g->Wid;
    Layout lq, lo;
    if ((rc = get_layout(lqkv, B, H, N, d, dt, "q/k/v", &lq)) != BLIN_OK) return rc;
    if ((rc = get_layout(lout, B, H, N, d, dt, "o", &lo)) != BLIN_OK) return rc;
    if ((rc = check_state(st)) != BLIN_OK) return rc;
    if (st->B != B || st->H != H || st->d != d)
        return fail(BLIN_ERR_STATE, "state is B=%d H=%d d=%d, call is B=%d H=%d d=%d", st->B, st->H, st->d,
                    B, H, d);
    if ((long long)st->t_next + frames >= (1LL << 30)) return fail(BLIN_ERR_SHAPE, "frame index overflow");
    // one causal block per call: the frames [t_next, t_next + frames) share block t_next / F
    if (st->t_next % F + frames > F)
        return fail(BLIN_ERR_SHAPE,
                    "frames [%d, %d) cross a block boundary (block_frames %d): a block step covers one block",
                    st->t_next, st->t_next + frames, F);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool tc = dt == BLIN_BF16 && tc_supported(d, g->rope_split);
    Plan p = make_plan(B, H, d, frames, g->Hgt, g->Wid, frames, st->t_next, true, g->rope_split, g->eps, tc);
    if ((rc = check_launch_limits(p)) != BLIN_OK) return rc;
    if (fp4 && !p.tc)
        return fail(BLIN_ERR_SHAPE, "NVFP4 inputs need the tensor-core path (rope split (8,12,12) at d=32 or "
                                    "(16,24,24) at d=64, and a RoPE table that fits shared memory)");
    p.g.lq = lq;
    p.g.lo = lo;
    if ((rc = ensure_scratch(st, plan_bytes(p), s)) != BLIN_OK) return rc;
    plan_bind(p, st->scratch);
    rc = run(p, q, k, v, o, dt, st->S, st->z, commit ? st->S : nullptr, commit ? st->z : nullptr,
             (double)g->theta, s, fp4);
    if (rc != BLIN_OK) return rc;
    if ((rc = mark_state_use(st, s)) != BLIN_OK) return rc;
    if (commit) st->t_next += frames;
    return BLIN_OK;
}

blin_status blin_prefill(const void *q, const void *k, const void *v, void *o, blin_dtype dt, int B, int H, int d,
                         const blin_geom *g, blin_state *st, void *workspace, size_t ws_bytes, blin_stream stream) {
    return prefill_impl(q, k, v, o, dt, B, H, d, g, nullptr, nullptr, st, workspace, ws_bytes, stream);
}

blin_status blin_prefill_strided(const void *q, const void *k, const void *v, void *o, blin_dtype dt, int B, int H,
                                 int d, const blin_geom *g, const blin_layout *qkv_layout,
                                 const blin_layout *o_layout, blin_state *st, void *workspace, size_t ws_bytes,
                                 blin_stream stream) {
    return prefill_impl(q, k, v, o, dt, B, H, d, g, qkv_layout, o_layout, st, workspace, ws_bytes, stream);
}

// NVFP4 operand checks: data and scale 16-byte aligned, positive finite global scale.
static blin_status check_fp4(const blin_nvfp4 *x, const char *name) {
    if (x == nullptr || x->data == nullptr || x->scale == nullptr)
        return fail(BLIN_ERR_INVALID_ARG, "NVFP4 %s: operand, data and scale must be non-NULL", name);
    if (!aligned16(x->data) || !aligned16(x->scale))
        return fail(BLIN_ERR_ALIGN, "NVFP4 %s: data and scale must be 16-byte aligned", name);
    if (!(x->global_scale > 0.f) || !std::isfinite(x->global_scale))
        return fail(BLIN_ERR_INVALID_ARG, "NVFP4 %s: global scale must be finite and > 0", name);
    return BLIN_OK;
}

blin_status blin_prefill_nvfp4(const blin_nvfp4 *q, const blin_nvfp4 *k, const blin_nvfp4 *v, void *o, int B, int H,
                               int d, const blin_geom *g, blin_state *st, void *workspace, size_t ws_bytes,
                               blin_stream stream) {
    blin_status rc;
    if ((rc = check_fp4(q, "q")) != BLIN_OK || (rc = check_fp4(k, "k")) != BLIN_OK || (rc = check_fp4(v, "v")) != BLIN_OK)
        return rc;
    const Fp4In fp4{q, k, v};
    return prefill_impl(q->data, k->data, v->data, o, BLIN_BF16, B, H, d, g, nullptr, nullptr, st, workspace, ws_bytes,
                        stream, &fp4);
}

blin_status blin_block_step_nvfp4(const blin_nvfp4 *q, const blin_nvfp4 *k, const blin_nvfp4 *v, void *o, int B,
                                  int H, int d, const blin_geom *g, blin_state *st, int commit, blin_stream stream) {
    blin_status rc;
    if ((rc = check_fp4(q, "q")) != BLIN_OK || (rc = check_fp4(k, "k")) != BLIN_OK || (rc = check_fp4(v, "v")) != BLIN_OK)
        return rc;
    const Fp4In fp4{q, k, v};
    return block_step_impl(q->data, k->data, v->data, o, BLIN_BF16, B, H, d, g, nullptr, nullptr, st, commit, stream,
                           &fp4);
}

blin_status blin_block_step(const void *q, const void *k, const void *v, void *o, blin_dtype dt, int B, int H,
                            int d, const blin_geom *g, blin_state *st, int commit, blin_stream stream) {
    return block_step_impl(q, k, v, o, dt, B, H, d, g, nullptr, nullptr, st, commit, stream);
}

blin_status blin_block_step_strided(const void *q, const void *k, const void *v, void *o, blin_dtype dt, int B,
                                    int H, int d, const blin_geom *g, const blin_layout *qkv_layout,
                                    const blin_layout *o_layout, blin_state *st, int commit, blin_stream stream) {
    return block_step_impl(q, k, v, o, dt, B, H, d, g, qkv_layout, o_layout, st, commit, stream);
}

int blin_last_path(void) { return g_last_path; }

blin_status blin_set_timing_events(void *const *events, int n) {
    if (events != nullptr && n < 8) return fail(BLIN_ERR_INVALID_ARG, "need 8 events (got %d)", n);
    g_timing = reinterpret_cast<cudaEvent_t const *>(events);
    return BLIN_OK;
}

unsigned long long blin_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

blin_status blin_device_status(int *code) {
    int c = 0;
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "device synchronise");
    e = read_and_clear_watchdog(&c);
    if (e != cudaSuccess) return cuda_fail(e, "watchdog read");
    if (code) *code = c;
    if (c != 0) return fail(BLIN_ERR_DEVICE, "a kernel wait ran out (watchdog code %d)", c);
    return BLIN_OK;
}

}  // extern "C"
