// Tensor-core path for bf16 Q/K/V on sm_100a (d = 32 or 64).
//
// Pass 1, partial_tc_kernel: per chunk (<= 1024 tokens of one block of one
//   head) the partial states P = sum (R_m phi(k_m)) v_m^T and zp = sum phi(k_m)
//   from one contraction
//       [K~^T ; phi(K)^T] x [V | 1]      (tcgen05.mma, fp32 in TMEM)
//   whose operands are MN-major views of the token-major tiles.
// Pass 2, output_tc_kernel: per group of <= 8 query tiles of one block of one
//   head, numerator and denominator from one contraction
//       [Q~ | phi(Q)] x [[S, 0], [0, z_hi z_lo]] = [num | phi(q).z_hi | phi(q).z_lo]
//   then o = num / (phi(q).z + eps) in fp32, stored as bf16.
//
// Both kernels are persistent (one CTA per SM) and split into roles (TMA
// producer, transform warps, one MMA-issuing thread, epilogue) that hand tiles
// to each other through mbarrier rings only; each CTA runs two such pipelines
// at d = 32 (see the pass 1 comment for why).  Every wait is bounded
// (ptx::mbar_wait_bounded), and work is ordered chunk-index major so the
// short last chunks of every block run last.
#pragma once

#include <cuda_bf16.h>

#include "blin_internal.cuh"
#include "ptx_sm100.cuh"

namespace blin {

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s: far beyond any legitimate wait

// Byte offset of 16-byte chunk `j` of row `r` inside a swizzled tile whose base
// is 1024-byte aligned (64B swizzle: rows of 64 B; 128B swizzle: rows of 128 B).
template <int D>
__device__ __forceinline__ uint32_t swz_chunk(int r, int j) {
    if constexpr (D == 32)
        return static_cast<uint32_t>(r * 64 + ((j ^ ((r >> 1) & 3)) << 4));
    else
        return static_cast<uint32_t>(r * 128 + ((j ^ (r & 7)) << 4));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Token position bookkeeping: relative frame t, row y, column x of a token,
// advanced by whole tiles without divisions.
struct TokPos {
    int t, y, x;
    __device__ __forceinline__ void init(const KGeom &g, int n) {
        t = n / g.HW;
        const int rem = n - t * g.HW;
        y = rem / g.Wg;
        x = rem - y * g.Wg;
    }
    __device__ __forceinline__ void advance(const KGeom &g, int dx, int dy, int dt) {
        x += dx;
        if (x >= g.Wg) { x -= g.Wg; ++y; }
        y += dy;
        if (y >= g.Hg) { y -= g.Hg; ++t; }
        t += dt;
    }
};

// A CTA's shared-memory RoPE table: (cos, sin) of every (position, pair) of
// the call's frame window and of every row and column, one section per axis.
// Each section is stored pair-major ([pair][position]) so that the threads of
// a warp, which hold consecutive tokens and hence mostly consecutive columns,
// read consecutive words: no bank conflicts on the x section, broadcasts on t, y.
struct RopeTab {
    const float2 *t, *y, *x;  // t indexed by relative frame (window offset folded in)
    int nt, ny, nx;            // positions per pair in each section (T, Hg, Wg)
};

// Fills this CTA's shared-memory RoPE table (the tensor-core path is only
// chosen when it fits; transform threads only, a barrier among them must
// follow).  Entry values are those of rope_entry (same order of operations).
template <int PT, int PY, int PX>
__device__ __forceinline__ RopeTab load_rope_tab(const KGeom &g, float2 *s_tab, int tid, int nthreads) {
    const int nt = g.T * PT, ny = g.Hg * PY, n = nt + ny + g.Wg * PX;
    for (int i = tid; i < n; i += nthreads) {
        int src;  // index of the same entry in the position-major order rope_entry enumerates
        if (i < nt) {
            src = (i % g.T) * PT + i / g.T;
        } else if (i < nt + ny) {
            const int r = i - nt;
            src = nt + (r % g.Hg) * PY + r / g.Hg;
        } else {
            const int r = i - nt - ny;
            src = nt + ny + (r % g.Wg) * PX + r / g.Wg;
        }
        s_tab[i] = rope_entry(src, g.T, g.t0, g.Hg, PT, PY, PX, g.theta);
    }
    RopeTab r;
    r.t = s_tab;
    r.y = s_tab + g.tab_y;
    r.x = s_tab + g.tab_x;
    r.nt = g.T;
    r.ny = g.Hg;
    r.nx = g.Wg;
    return r;
}

// phi (ReLU) then 3D RoPE of one token row held as D/2 bf16x2 words (pair p =
// features 2p, 2p+1, low half = even feature).  Writes phi into `ph` (bf16x2,
// exact) and optionally sums phi into zp.
// (RoPE inside linear attention: talk transcript; RoPE only in the numerator:
// news article, positional-encoding paragraph.)
template <int D, int PT, int PY, int PX, bool ZP>
__device__ __forceinline__ void phi_rope_row(uint32_t (&w)[D / 2], uint32_t (&ph)[D / 2], const RopeTab &tab,
                                             const TokPos &tp, float *zp) {
    static_assert(PT + PY + PX == D / 2, "split must cover d");
    const float2 *rt = tab.t + tp.t;
    const float2 *ry = tab.y + tp.y;
    const float2 *rx = tab.x + tp.x;
#pragma unroll
    for (int p = 0; p < D / 2; ++p) {
        const float2 cs = p < PT ? rt[p * tab.nt] : (p < PT + PY ? ry[(p - PT) * tab.ny] : rx[(p - PT - PY) * tab.nx]);
        // ReLU on the packed pair (exact), then widen
        __nv_bfloat162 hv = *reinterpret_cast<__nv_bfloat162 *>(&w[p]);
        hv = __hmax2(hv, __float2bfloat162_rn(0.f));
        const uint32_t u = *reinterpret_cast<uint32_t *>(&hv);
        ph[p] = u;
        const float a = __uint_as_float(u << 16);
        const float b = __uint_as_float(u & 0xFFFF0000u);
        if constexpr (ZP) {
            zp[2 * p] += a;
            zp[2 * p + 1] += b;
        }
        w[p] = pack_bf16x2(fmaf(a, cs.x, -b * cs.y), fmaf(a, cs.y, b * cs.x));
    }
}

template <int D>
__device__ __forceinline__ void load_row(const uint8_t *tile, int r, uint32_t (&w)[D / 2]) {
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
        const uint4 v = *reinterpret_cast<const uint4 *>(tile + swz_chunk<D>(r, j));
        w[4 * j + 0] = v.x;
        w[4 * j + 1] = v.y;
        w[4 * j + 2] = v.z;
        w[4 * j + 3] = v.w;
    }
}
template <int D>
__device__ __forceinline__ void store_row(uint8_t *tile, int r, const uint32_t (&w)[D / 2]) {
#pragma unroll
    for (int j = 0; j < D / 8; ++j)
        *reinterpret_cast<uint4 *>(tile + swz_chunk<D>(r, j)) =
            make_uint4(w[4 * j + 0], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
}
template <int D>
__device__ __forceinline__ void zero_row(uint8_t *tile, int r) {
#pragma unroll
    for (int j = 0; j < D / 8; ++j)
        *reinterpret_cast<uint4 *>(tile + swz_chunk<D>(r, j)) = make_uint4(0, 0, 0, 0);
}

// Rounds a pointer into the kernel's dynamic shared memory up to 1024 bytes by
// indexing from it (not through an integer cast), so the compiler keeps every
// derived access in the shared address space (LDS/STS, not generic loads).
__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    const uint32_t a = ptx::smem_u32(p);
    return p + ((1024u - (a & 1023u)) & 1023u);
}

// Loads `n` (1, 2 or 32) consecutive fp32 TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_ld_2cols(uint32_t taddr, float &a, float &b) {
    uint32_t r0, r1;
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0, %1}, [%2];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r0), "=r"(r1)
        : "r"(taddr)
        : "memory");
    a = __uint_as_float(r0);
    b = __uint_as_float(r1);
}

// ---------------------------------------------------------------------------- output B operand
template <int D>
struct OutB {  // the output kernel's B operand: K atoms of N rows, bf16, K-major, swizzled
    static constexpr int N = D + 16;          // num | phi.z_hi | phi.z_lo | zero pad
    static constexpr int ROWB = 2 * D;
    static constexpr int BATOM = N * ROWB;    // one K atom
    static constexpr int IMG = 2 * BATOM;     // atom 0: S part, atom 1: z part
};

template <int D>
__device__ __forceinline__ int swz_bits(int n) {
    return D == 32 ? ((n >> 1) & 3) : (n & 7);
}

// One 16-byte chunk (`item`, in storage order) of the B operand built from the
// fp32 prefix state `pre` (S row-major [key feature][value feature], then z):
// atom 0 row n < D holds S[.][n]; atom 1 rows D and D+1 hold z split into a
// bf16 high part and the bf16 rounding of the remainder; all else is zero.
template <int D>
__device__ __forceinline__ uint4 b_operand_chunk(const float *pre, int item) {
    using B = OutB<D>;
    const int atom = item / (B::BATOM / 16), rr = item % (B::BATOM / 16);
    const int n = rr / (D / 8), gq = (rr % (D / 8)) ^ swz_bits<D>(n);
    uint32_t w4[4] = {0u, 0u, 0u, 0u};
    if (atom == 0 && n < D) {
#pragma unroll
        for (int u = 0; u < 4; ++u) w4[u] = pack_bf16x2(pre[(8 * gq + 2 * u) * D + n], pre[(8 * gq + 2 * u + 1) * D + n]);
    } else if (atom == 1 && (n == D || n == D + 1)) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            float zz[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float z = pre[D * D + 8 * gq + 2 * u + h];
                const float hi = __bfloat162float(__float2bfloat16_rn(z));
                zz[h] = n == D ? hi : z - hi;
            }
            w4[u] = pack_bf16x2(zz[0], zz[1]);
        }
    }
    return make_uint4(w4[0], w4[1], w4[2], w4[3]);
}

// ============================================================================ shared control
__device__ __forceinline__ int ld_volatile(const int *p) { return *reinterpret_cast<const volatile int *>(p); }

// Each pipeline's producer ends its tile stream with this unit id in the
// landing-slot record; the transform warps pass it on to the MMA issuer through
// the operand ring, and both stop there.
constexpr int kEndFirst = -1;

// One mbarrier arrival for the whole warp, after every lane's shared-memory
// accesses (and tcgen05 loads, fenced by the caller) are ordered before it.
__device__ __forceinline__ void warp_arrive(uint32_t bar, int lane) {
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(bar);
}

// ============================================================================ pass 1
template <int D>
struct P1 {
    static constexpr int ROWB = 2 * D;
    static constexpr int TB = kTile * ROWB;
    static constexpr int M = D == 32 ? 64 : 128;          // [K~^T ; phi(K)^T]
    static constexpr int N = D == 32 ? D + 8 : D + 16;   // [V | ones]
    static constexpr int NP = D == 32 ? 2 : 1;           // independent pipelines per CTA (MMA issuers)
    static constexpr int NK = D == 32 ? 4 : 3;           // K landing slots per pipeline (free once read)
    static constexpr int NV = D == 32 ? 5 : 4;           // V landing slots per pipeline (free once the MMA is done)
    static constexpr int NO = 2;                         // operand sets per pipeline: K~ | phi
    static constexpr int NACC = 2;                       // TMEM accumulators per pipeline (chunks in flight)
    static constexpr int ACOLS = D == 32 ? 64 : 128;     // TMEM columns per accumulator
    static constexpr uint32_t TCOLS = NP * NACC * ACOLS;
    static constexpr uint32_t LAYOUT = D == 32 ? 4u : 2u;
    static constexpr int NBAR = 2 * NK + NV + NO + 2 * NACC;  // mbarriers per pipeline
    static constexpr int CTRL = 1024;
    static constexpr int BARS = 512;                     // mbarrier area at the start of the control block
    static constexpr int RINGS = NP * (2 * NO + NK + NV) * TB;  // operand, K and V rings of all pipelines
    static constexpr int FIXED = RINGS + TB + CTRL + 1024;  // + RoPE table
    static constexpr int THREADS = 32 * 6 * NP;  // warps [0, 4NP) transform, then NP producers, NP MMA issuers
    static_assert(NP * (NBAR + 1) * 8 <= BARS, "mbarriers (+ one drain barrier per pipeline) overflow their area");
    static_assert(BARS + 4 * NP * (4 * NK + 4 * NO) + 16 <= CTRL, "control block overflow");
    static_assert(NV > NO, "an operand slot's release is read from the V ring's tile-done barriers");
    // the B operand's second N atom (the ones block) sits above every V slot
    static_assert(NP * NV * TB < (1 << 18), "LBO field range");
    static_assert(TCOLS <= 512, "TMEM holds 512 columns");
};

// Persistent, one CTA per SM (a kernel that uses tcgen05 gets one CTA per SM).
// The CTA runs NP independent pipelines, so that NP threads issue MMAs: one
// thread issues a tcgen05.mma about every 50 cycles and the eight M = 64 MMAs
// a 128-token tile needs from one thread would not keep up with HBM, while two
// issuers' MMAs overlap in the tensor core.  Chunks are taken in
// chunk-index-major order (the short last chunk of every block comes last):
// pipeline p of CTA j first takes chunk j + p * grid, then the next unclaimed
// chunk from a work counter, so all pipelines finish within about one chunk.
// Per pipeline: a producer thread lands each K tile and V tile with TMA in
// two rings; four transform warps read K (its slot is free again at once) and
// write the A operand (K~, phi(K)) into an operand ring; an MMA thread
// accumulates [K~^T; phi^T] x [V | 1] into a TMEM accumulator per chunk,
// taking V straight from its landing slot, and commits once per tile to that V
// slot's tile-done barrier, which frees both the V slot and the tile's operand
// slot.  Two tiles into the next chunk, the transform warps read the finished
// accumulator back (each warp its TMEM subpartition) and write the chunk
// partial to global memory.
template <int D, int PT, int PY, int PX>
__global__ void __launch_bounds__(P1<D>::THREADS, 1)
    partial_tc_kernel(const __grid_constant__ CUtensorMap mk, const __grid_constant__ CUtensorMap mv,
                      KGeom g, int *watchdog) {
    using C = P1<D>;
    constexpr int NP = C::NP, NK = C::NK, NV = C::NV, NO = C::NO, NA = C::NACC, TB = C::TB, ROWB = C::ROWB,
                  E = D * D + D;
    constexpr uint32_t IDESC = ptx::idesc_bf16_f32(C::M, C::N, 1, 1);

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *opnd0 = smem;                         // [NP][NO][K~ | phi]
    uint8_t *kring0 = opnd0 + NP * NO * 2 * TB;    // [NP][NK][K]
    uint8_t *vring0 = kring0 + NP * NK * TB;       // [NP][NV][V]
    uint8_t *ones = vring0 + NP * NV * TB;         // constant B block (above every V tile: positive LBO)
    uint8_t *ctrl = ones + TB;
    volatile int *flags = reinterpret_cast<volatile int *>(ctrl + C::BARS);  // [0] abort
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(ctrl + C::BARS + 4);
    int *info0 = reinterpret_cast<int *>(ctrl + C::BARS + 16);          // [NP][NK + NO][4]
    float2 *s_tab = reinterpret_cast<float2 *>(ctrl + C::CTRL);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // this thread's pipeline
    const int pipe = warp < 4 * NP ? warp >> 2 : (warp - 4 * NP) % NP;
    uint8_t *kring = kring0 + pipe * NK * TB;
    uint8_t *vring = vring0 + pipe * NV * TB;
    uint8_t *opnd = opnd0 + pipe * NO * 2 * TB;
    uint64_t *bars = reinterpret_cast<uint64_t *>(ctrl) + pipe * C::NBAR;
    int *linfo = info0 + pipe * 4 * (NK + NO);  // [NK][4] unit, tile, valid, last
    int *oinfo = linfo + 4 * NK;                 // [NO][4]
    auto lk = [&](int s) { return kring + s * TB; };
    auto lv = [&](int s) { return vring + s * TB; };
    auto ok_ = [&](int s) { return opnd + s * 2 * TB; };
    auto op_ = [&](int s) { return opnd + s * 2 * TB + TB; };
    // kfull[s]: K and V of the tile in K slot s have landed (TMA bytes);
    // kempty[s]: its K has been read (4 transform warps);
    // tdone[s]: the MMAs of the tile in V slot s are done (1 commit): V slot s
    //   and that tile's operand slot are free;
    // ofull[s]: operand slot s is written (4 transform warps)
    auto kfull = [&](int s) { return ptx::smem_u32(bars + s); };
    auto kempty = [&](int s) { return ptx::smem_u32(bars + NK + s); };
    auto tdone = [&](int s) { return ptx::smem_u32(bars + 2 * NK + s); };
    auto ofull = [&](int s) { return ptx::smem_u32(bars + 2 * NK + NV + s); };
    auto accf = [&](int a) { return ptx::smem_u32(bars + 2 * NK + NV + NO + a); };
    auto acce = [&](int a) { return ptx::smem_u32(bars + 2 * NK + NV + NO + NA + a); };
    // drain: one final commit, so that the MMA thread leaves only after all its MMAs are done
    const uint32_t drain = ptx::smem_u32(reinterpret_cast<uint64_t *>(ctrl) + NP * C::NBAR + pipe);

    const int units = g.cpb * g.nblk * g.BH;
    const int per_c = g.nblk * g.BH;
    // chunk-index-major order: the short last chunks of every block come last
    auto decode = [&](int u, int &bh, int &b, int &c) {
        c = u / per_c;
        const int rem = u - c * per_c;
        bh = rem / g.nblk;
        b = rem - bh * g.nblk;
    };

    if (tid == 0) {
        for (int p = 0; p < NP; ++p) {
            uint64_t *pb = reinterpret_cast<uint64_t *>(ctrl) + p * C::NBAR;
            for (int s = 0; s < NK; ++s) {
                ptx::mbar_init(ptx::smem_u32(pb + s), 1);            // kfull: producer (+ TMA bytes)
                ptx::mbar_init(ptx::smem_u32(pb + NK + s), 4);       // kempty: one arrival per transform warp
            }
            for (int s = 0; s < NV; ++s) ptx::mbar_init(ptx::smem_u32(pb + 2 * NK + s), 1);       // tdone: commit
            for (int s = 0; s < NO; ++s) ptx::mbar_init(ptx::smem_u32(pb + 2 * NK + NV + s), 4);  // ofull
            for (int a = 0; a < NA; ++a) {
                ptx::mbar_init(ptx::smem_u32(pb + 2 * NK + NV + NO + a), 1);       // accf: commit
                ptx::mbar_init(ptx::smem_u32(pb + 2 * NK + NV + NO + NA + a), 4);  // acce: transform warps
            }
            ptx::mbar_init(ptx::smem_u32(reinterpret_cast<uint64_t *>(ctrl) + NP * C::NBAR + p), 1);  // drain
        }
        flags[0] = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 0) {
        ptx::tmem_alloc(ptx::smem_u32(tmem_slot), C::TCOLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot + pipe * NA * C::ACOLS;  // this pipeline's accumulators
    if (tid == 0) griddep_launch_dependents();

    if (warp >= 4 * NP && warp < 5 * NP) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            ptx::tma_prefetch_map(&mk);
            ptx::tma_prefetch_map(&mv);
            const uint64_t stream_policy = ptx::l2_evict_first();  // K and V are read once
            int k = 0;
            bool ok = true;
            // the first NP * grid chunks are dealt out statically (chunk blockIdx.x + pipe * grid); after
            // that each pipeline takes the next unclaimed chunk from a counter, in chunk-index-major
            // order, so the long chunks go first and every pipeline ends within about one chunk of the
            // others.  The claim for the following chunk is issued a chunk ahead (its latency hidden).
            const int first_dyn = NP * gridDim.x;
            int next = first_dyn + static_cast<int>(atomicAdd(g.sched, 1u));
            for (int u = blockIdx.x + pipe * gridDim.x; ok && u < units;) {
                const int u_next = next;
                if (u_next < units) next = first_dyn + static_cast<int>(atomicAdd(g.sched, 1u));
                int bh, b, c;
                decode(u, bh, b, c);
                const int fb = block_frame_begin(g, b), fe = block_frame_end(g, b);
                const int bntok = (fe - fb) * g.HW, cs = c * kChunk;
                if (cs < bntok) {
                    const int clen = min(kChunk, bntok - cs), ntiles = (clen + kTile - 1) / kTile;
                    const int row0 = bh * g.N + fb * g.HW + cs;
                    for (int t = 0; t < ntiles; ++t, ++k) {
                        const int sk = k % NK, sv = k % NV;
                        if ((k >= NK && !ptx::mbar_wait_bounded(kempty(sk), ((k / NK) - 1) & 1, watchdog,
                                                                WD_PARTIAL_EMPTY, kWaitLimitNs)) ||
                            (k >= NV && !ptx::mbar_wait_bounded(tdone(sv), ((k / NV) - 1) & 1, watchdog,
                                                                WD_PARTIAL_EMPTY, kWaitLimitNs))) {
                            ok = false;
                            break;
                        }
                        int *inf = linfo + 4 * sk;
                        inf[0] = u;
                        inf[1] = t;
                        inf[2] = min(kTile, clen - t * kTile);
                        inf[3] = t == ntiles - 1;
                        ptx::mbar_arrive_expect_tx(kfull(sk), 2 * TB);
                        ptx::tma_load_2d_hint(ptx::smem_u32(lk(sk)), &mk, kfull(sk), 0, row0 + t * kTile, stream_policy);
                        ptx::tma_load_2d_hint(ptx::smem_u32(lv(sv)), &mv, kfull(sk), 0, row0 + t * kTile, stream_policy);
                    }
                }
                u = u_next;
            }
            // end marker for the transform warps
            const int sk = k % NK;
            if (ok && (k < NK || ptx::mbar_wait_bounded(kempty(sk), ((k / NK) - 1) & 1, watchdog, WD_PARTIAL_EMPTY,
                                                        kWaitLimitNs))) {
                linfo[4 * sk] = kEndFirst;
                ptx::mbar_arrive(kfull(sk));
            }
        }
    } else if (warp >= 5 * NP) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int nu = 0;
            for (int k = 0;; ++k) {
                const int so = k % NO;
                if (flags[0] ||
                    !ptx::mbar_wait_bounded(ofull(so), (k / NO) & 1, watchdog, WD_PARTIAL_READY, kWaitLimitNs)) {
                    flags[0] = 1;
                    break;
                }
                const int *inf = oinfo + 4 * so;
                const int u = ld_volatile(inf), t = ld_volatile(inf + 1), last = ld_volatile(inf + 3);
                if (u < 0) break;
                const int a = nu % NA;
                if (t == 0 && nu >= NA &&
                    !ptx::mbar_wait_bounded(acce(a), ((nu / NA) - 1) & 1, watchdog, WD_PARTIAL_ACC, kWaitLimitNs)) {
                    flags[0] = 1;
                    break;
                }
                ptx::tc_fence_after_sync();
                const int sv = k % NV;  // the tile's V slot (same tile order as the producer)
                const uint32_t va = ptx::smem_u32(lv(sv));
                // A (MN-major): M atom 0 = K~ rows, atom 1 (+TB) = phi rows; B: V | ones.
                // Consecutive K steps are 16 token rows (16 * ROWB bytes: ROWB in the address field).
                const uint64_t ad = ptx::smem_desc(ptx::smem_u32(ok_(so)), TB, 8 * ROWB, C::LAYOUT);
                const uint64_t bd = ptx::smem_desc(va, ptx::smem_u32(ones) - va, 8 * ROWB, C::LAYOUT);
                const uint32_t dacc = tmem + a * C::ACOLS;
#pragma unroll
                for (int kk = 0; kk < kTile / 16; ++kk)
                    ptx::mma_bf16_ss(dacc, ad + static_cast<uint64_t>(kk * ROWB), bd + static_cast<uint64_t>(kk * ROWB),
                                     IDESC, (t > 0 || kk > 0) ? 1u : 0u);
                ptx::mma_commit(tdone(sv));
                if (last) {
                    ptx::mma_commit(accf(a));
                    ++nu;
                }
            }
            // every MMA (and the arrivals of the commits above) completes before the CTA's
            // final barrier and TMEM release, also when a wait gave up
            ptx::mma_commit(drain);
            if (!ptx::mbar_wait_bounded(drain, 0, watchdog, WD_PARTIAL_ACC, kWaitLimitNs)) flags[0] = 1;
        }
    } else {
        // ------------------------------------------------------------ transform warps: one row per thread
        const int r = tid & 127, sub = warp & 3;
        const RopeTab tab = load_rope_tab<PT, PY, PX>(g, s_tab, tid, 128 * NP);
        {
            uint4 *o4 = reinterpret_cast<uint4 *>(ones);  // all 1.0, so its swizzle is irrelevant
            for (int i = tid; i < TB / 16; i += 128 * NP) o4[i] = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
        }
        ptx::fence_proxy_async_smem();  // the ones block is read by the MMA (async proxy)
        ptx::named_bar_sync(1, 128 * NP);

        // Chunk epilogue (each warp its TMEM subpartition): accumulator -> chunk
        // partial.  M = 64 (d = 32): accumulator row m in TMEM lane
        // (m % 16) + 32 * (m / 16); M = 128 (d = 64): row m in lane m.  Rows
        // [0, D) hold P, rows [D, 2D) hold phi^T against the ones block, i.e. zp,
        // in column D.
        auto epilogue = [&](int u, int a, int ph) {
            if (!ptx::mbar_wait_bounded(accf(a), ph, watchdog, WD_PARTIAL_ACC, kWaitLimitNs)) flags[0] = 1;
            ptx::tc_fence_after_sync();
            constexpr int RPS = D == 32 ? 16 : 32;  // accumulator rows per TMEM subpartition
            int bh, b, c;
            decode(u, bh, b, c);
            float *out = g.part + ((size_t)(bh * g.nblk + b) * g.cpb + c) * E;
            const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * sub) << 16) + a * C::ACOLS;
            if (sub < 2) {
                const int m = RPS * sub + lane;  // P row
#pragma unroll
                for (int half = 0; half < D / 32; ++half) {
                    float v[32];
                    ptx::tmem_ld_32cols(taddr + 32 * half, v);
                    if (lane < RPS) {
                        float4 *dst = reinterpret_cast<float4 *>(out + m * D + 32 * half);
#pragma unroll
                        for (int j = 0; j < 8; ++j) dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
                    }
                }
            } else {
                float zv, unused;
                tmem_ld_2cols(taddr + D, zv, unused);
                if (lane < RPS) out[D * D + RPS * (sub - 2) + lane] = zv;
            }
            ptx::tc_fence_before_sync();
            warp_arrive(acce(a), lane);  // accumulator a is free again
        };

        const int dx = kTile % g.Wg, dy = (kTile / g.Wg) % g.Hg, dt = kTile / g.HW;
        TokPos tp{0, 0, 0};
        int nu = 0;                               // chunks pushed to the MMA so far
        int pend_u = -1, pend_a = 0, pend_ph = 0;  // finished chunk whose epilogue is still due
        int since = 0;                            // tiles pushed since that chunk's last tile
        for (int k = 0;; ++k) {
            const int sk = k % NK, so = k % NO;
            if (flags[0] || !ptx::mbar_wait_bounded(kfull(sk), (k / NK) & 1, watchdog, WD_PARTIAL_FULL, kWaitLimitNs)) {
                flags[0] = 1;
                break;
            }
            const int *inf = linfo + 4 * sk;
            const int u = ld_volatile(inf), t = ld_volatile(inf + 1), valid = ld_volatile(inf + 2);
            const int last = ld_volatile(inf + 3);
            // read this row of K; rows past the chunk also clear their V row
            // (the MMA reads V in place: other blocks' tokens must add nothing)
            uint32_t w[D / 2], ph[D / 2];
            const bool live = u >= 0 && r < valid;
            if (live) load_row<D>(lk(sk), r, w);
            else if (u >= 0) zero_row<D>(lv(k % NV), r);
            // the next TMA into this K slot writes through the async proxy: order
            // this thread's generic reads of the slot before it
            ptx::fence_proxy_async_smem();
            if (u >= 0) warp_arrive(kempty(sk), lane);
            // operand slot so was last used by tile k - NO: wait for its MMAs
            if (k >= NO && !ptx::mbar_wait_bounded(tdone((k - NO) % NV), ((k - NO) / NV) & 1, watchdog,
                                                   WD_PARTIAL_READY, kWaitLimitNs)) {
                flags[0] = 1;
                break;
            }
            if (u < 0) {  // pass the end on to the MMA issuer, in operand order
                if (r == 0) oinfo[4 * so] = kEndFirst;
                warp_arrive(ofull(so), lane);
                break;
            }
            if (t == 0) {
                int bh, b, c;
                decode(u, bh, b, c);
                tp.init(g, block_frame_begin(g, b) * g.HW + c * kChunk + r);
            } else {
                tp.advance(g, dx, dy, dt);
            }
            if (live) {
                phi_rope_row<D, PT, PY, PX, false>(w, ph, tab, tp, nullptr);
                store_row<D>(ok_(so), r, w);
                store_row<D>(op_(so), r, ph);
            } else {  // rows past the chunk add nothing
                zero_row<D>(ok_(so), r);
                zero_row<D>(op_(so), r);
            }
            ptx::fence_proxy_async_smem();
            if (r == 0) {
                int *oi = oinfo + 4 * so;
                oi[0] = u;
                oi[1] = t;
                oi[2] = valid;
                oi[3] = last;
            }
            warp_arrive(ofull(so), lane);
            // the previous chunk's epilogue, once its MMAs have had two tiles' time
            if (pend_u >= 0 && (++since >= 2 || last)) {
                epilogue(pend_u, pend_a, pend_ph);
                pend_u = -1;
            }
            if (last) {
                pend_u = u;
                pend_a = nu % NA;
                pend_ph = (nu / NA) & 1;
                since = 0;
                ++nu;
            }
        }
        if (pend_u >= 0 && !flags[0]) epilogue(pend_u, pend_a, pend_ph);
    }
    ptx::tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after_sync();
        ptx::tmem_dealloc(*tmem_slot, C::TCOLS);
    }
}

// ============================================================================ pass 2
template <int D>
struct P2 {
    static constexpr int ROWB = 2 * D;
    static constexpr int TB = kTile * ROWB;
    static constexpr int NP = D == 32 ? 2 : 1;          // independent pipelines per CTA (MMA issuers)
    static constexpr int NL = D == 32 ? 6 : 3;          // Q landing slots per pipeline
    static constexpr int NO = 2;                        // operand sets per pipeline: q~ | phi(q)
    static constexpr int NACC = 4;                      // TMEM accumulators per pipeline
    static constexpr int NT = NACC > NO + 1 ? NACC : NO + 1;  // tile-done barriers per pipeline
    static constexpr int N = OutB<D>::N;                // num | phi.z_hi | phi.z_lo | pad
    static constexpr int BATOM = OutB<D>::BATOM;        // one K atom of B (N rows)
    static constexpr int IMG = OutB<D>::IMG;
    static constexpr int ACOLS = D == 32 ? 64 : 128;    // TMEM columns per accumulator
    static constexpr uint32_t TCOLS = NP * NACC * ACOLS;
    static constexpr uint32_t LAYOUT = D == 32 ? 4u : 2u;
    static constexpr int PRE = (D * D + D) * 4;         // one fp32 prefix state (S, z)
    static constexpr int NBAR = 2 * NL + NO + NT + NACC + 6;  // + pfull, pempty, bempty (2 each)
    static constexpr int CTRL = 2048;
    static constexpr int BARS = 512;
    // shared memory of one pipeline, rounded up so every pipeline's swizzled
    // tiles stay 1024-byte aligned
    // (+ TB: each epilogue warp's 32-row O staging area for its TMA store)
    // (the fp32 prefix state is single-buffered: it is turned into the
    // double-buffered bf16 B operand as soon as it lands)
    static constexpr int PIPE = (NL * TB + NO * 2 * TB + TB + 2 * IMG + PRE + 1023) / 1024 * 1024;
    static constexpr int FIXED = NP * PIPE + CTRL + 1024;  // + RoPE table
    static constexpr int THREADS = 32 * 10 * NP;  // per pipeline: 4 transform, 4 epilogue, producer, MMA warps
    static_assert(NP * (NBAR + 1) * 8 <= BARS, "mbarriers (+ one drain barrier per pipeline) overflow their area");
    static_assert(BARS + 16 + NP * 4 * 8 * (NL + NO) <= CTRL, "control block overflow");
    static_assert(TCOLS <= 512, "TMEM holds 512 columns");
    static_assert(PIPE % 1024 == 0, "pipelines keep 1024-byte alignment");
};

// Persistent, one CTA per SM, NP independent pipelines (see pass 1: two
// issuing threads keep the tensor core fed).  Pipeline p takes every other
// group of <= 8 query tiles of one (head, block) from the CTA's static round
// robin.  Per pipeline: a producer thread bulk-copies each group's fp32
// prefix state and lands its Q tiles with TMA; four transform warps build the
// group's bf16 B operand [[S, 0], [0, z_hi z_lo]] from the prefix state, then
// write [R phi(q) | phi(q)] per tile into an operand ring; an MMA thread
// computes [Q~ | phi(Q)] x B into one of NACC TMEM accumulators and commits
// once per tile to a tile-done barrier (which frees the operand slot and tells
// the epilogue the accumulator is ready); four epilogue warps divide
// num / (phi(q).z + eps) in fp32, free the accumulator, and each stages its 32
// bf16 rows in shared memory and stores them with its own TMA store (plain
// stores for the warp that holds a ragged tile's edge).  `mo` views O with
// 32-row boxes.
template <int D, int PT, int PY, int PX>
__global__ void __launch_bounds__(P2<D>::THREADS, 1)
    output_tc_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mo, KGeom g,
                     __nv_bfloat16 *o, int *watchdog) {
    using C = P2<D>;
    constexpr int NP = C::NP, NL = C::NL, NO = C::NO, NA = C::NACC, NT = C::NT, TB = C::TB, ROWB = C::ROWB;
    constexpr uint32_t IDESC = ptx::idesc_bf16_f32(128, C::N, 0, 0);
    const int QG = g.qgt * kTile;  // tokens per group

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *ctrl = smem + NP * C::PIPE;
    volatile int *flags = reinterpret_cast<volatile int *>(ctrl + C::BARS);  // [0] abort
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(ctrl + C::BARS + 4);
    float2 *s_tab = reinterpret_cast<float2 *>(ctrl + C::CTRL);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // roles: warps [0, 4NP) transform, [4NP, 8NP) epilogue, then NP producers, NP MMA issuers
    const int pipe = warp < 8 * NP ? (warp >> 2) % NP : (warp - 8 * NP) % NP;
    uint8_t *pb = smem + pipe * C::PIPE;
    uint8_t *land = pb;                           // [NL][Q]
    uint8_t *opnd = land + NL * TB;               // [NO][q~ | phi]
    uint8_t *ostg = opnd + NO * 2 * TB;           // [4 warps][32 rows] O staging
    uint8_t *bbuf = ostg + TB;                    // [2][IMG] bf16 B operand
    uint8_t *pbuf = bbuf + 2 * C::IMG;            // [PRE] fp32 prefix state
    uint64_t *bars = reinterpret_cast<uint64_t *>(ctrl) + pipe * C::NBAR;
    int *linfo = reinterpret_cast<int *>(ctrl + C::BARS + 16) + pipe * 8 * (NL + NO);  // [NL][8]
    int *oinfo = linfo + 8 * NL;                                                     // [NO][8]
    auto lq = [&](int s) { return land + s * TB; };
    auto oq = [&](int s) { return opnd + s * 2 * TB; };
    auto oph = [&](int s) { return opnd + s * 2 * TB + TB; };
    auto lfull = [&](int s) { return ptx::smem_u32(bars + s); };
    auto lempty = [&](int s) { return ptx::smem_u32(bars + NL + s); };
    auto ofull = [&](int s) { return ptx::smem_u32(bars + 2 * NL + s); };
    auto tdone = [&](int s) { return ptx::smem_u32(bars + 2 * NL + NO + s); };
    auto acce = [&](int a) { return ptx::smem_u32(bars + 2 * NL + NO + NT + a); };
    auto pfull = [&](int s) { return ptx::smem_u32(bars + 2 * NL + NO + NT + NA + s); };
    auto pempty = [&](int s) { return ptx::smem_u32(bars + 2 * NL + NO + NT + NA + 2 + s); };
    auto bempty = [&](int s) { return ptx::smem_u32(bars + 2 * NL + NO + NT + NA + 4 + s); };
    // drain: one final commit, so that the MMA thread leaves only after all its MMAs are done
    const uint32_t drain = ptx::smem_u32(reinterpret_cast<uint64_t *>(ctrl) + NP * C::NBAR + pipe);

    const int units = g.qcpb * g.nblk * g.BH;
    const int per_q = g.nblk * g.BH;
    auto decode = [&](int u, int &bh, int &b, int &qc) {
        qc = u / per_q;
        const int rem = u - qc * per_q;
        bh = rem / g.nblk;
        b = rem - bh * g.nblk;
    };

    if (tid == 0) {
        for (int p = 0; p < NP; ++p) {
            uint64_t *bp = reinterpret_cast<uint64_t *>(ctrl) + p * C::NBAR;
            for (int s = 0; s < NL; ++s) {
                ptx::mbar_init(ptx::smem_u32(bp + s), 1);       // lfull: producer + TMA bytes
                ptx::mbar_init(ptx::smem_u32(bp + NL + s), 4);  // lempty: transform warps
            }
            for (int s = 0; s < NO; ++s) ptx::mbar_init(ptx::smem_u32(bp + 2 * NL + s), 4);           // ofull
            for (int s = 0; s < NT; ++s) ptx::mbar_init(ptx::smem_u32(bp + 2 * NL + NO + s), 1);      // tdone
            for (int a = 0; a < NA; ++a) ptx::mbar_init(ptx::smem_u32(bp + 2 * NL + NO + NT + a), 4);  // acce
            for (int s = 0; s < 2; ++s) {
                ptx::mbar_init(ptx::smem_u32(bp + 2 * NL + NO + NT + NA + s), 1);      // pfull: bulk copy
                ptx::mbar_init(ptx::smem_u32(bp + 2 * NL + NO + NT + NA + 2 + s), 4);  // pempty: transform warps
                ptx::mbar_init(ptx::smem_u32(bp + 2 * NL + NO + NT + NA + 4 + s), 1);  // bempty: commit
            }
            ptx::mbar_init(ptx::smem_u32(reinterpret_cast<uint64_t *>(ctrl) + NP * C::NBAR + p), 1);  // drain
        }
        flags[0] = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 0) {
        ptx::tmem_alloc(ptx::smem_u32(tmem_slot), C::TCOLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot + pipe * NA * C::ACOLS;  // this pipeline's accumulators

    // this pipeline's groups: units blockIdx.x + (pipe + NP j) * gridDim.x
    const int u0 = blockIdx.x + pipe * gridDim.x, ustep = NP * gridDim.x;

    if (warp >= 8 * NP && warp < 9 * NP) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            ptx::tma_prefetch_map(&mq);
            const uint64_t stream_policy = ptx::l2_evict_first();  // Q is read once
            int k = 0, nu = 0;
            bool waited = false, ok = true;
            auto issue_prefix = [&](int bh, int b, int ord) {
                // the previous group's prefix has been turned into its B operand
                if (ord >= 1 &&
                    !ptx::mbar_wait_bounded(pempty(0), (ord - 1) & 1, watchdog, WD_OUT_BREADY, kWaitLimitNs))
                    return false;
                if (!waited) {  // the prefix states are written by the scan
                    griddep_wait();
                    waited = true;
                }
                ptx::mbar_arrive_expect_tx(pfull(0), C::PRE);
                ptx::bulk_load(ptx::smem_u32(pbuf), g.prefix + ((size_t)bh * g.nblk + b) * (D * D + D), C::PRE,
                               pfull(0));
                return true;
            };
            for (int u = u0; ok && u < units; u += ustep) {
                int bh, b, qc;
                decode(u, bh, b, qc);
                const int fb = block_frame_begin(g, b), fe = block_frame_end(g, b);
                const int bntok = (fe - fb) * g.HW, qs = qc * QG;
                if (qs >= bntok) continue;
                const int qlen = min(QG, bntok - qs), ntiles = (qlen + kTile - 1) / kTile;
                const int row0 = bh * g.N + fb * g.HW + qs;
                // the first group's Q tiles go out before waiting on the scan
                const int early = waited ? 0 : min(ntiles, NL);
                if (early == 0 && !(ok = issue_prefix(bh, b, nu))) break;
                for (int t = 0; t < ntiles; ++t, ++k) {
                    const int sl = k % NL;
                    if (k >= NL &&
                        !ptx::mbar_wait_bounded(lempty(sl), ((k / NL) - 1) & 1, watchdog, WD_OUT_EMPTY, kWaitLimitNs)) {
                        ok = false;
                        break;
                    }
                    int *inf = linfo + 8 * sl;
                    inf[0] = u;
                    inf[1] = t;
                    inf[2] = min(kTile, qlen - t * kTile);
                    inf[3] = nu;
                    inf[4] = fb * g.HW + qs;  // token index (within the head) of the group's first row
                    inf[5] = t == ntiles - 1;
                    ptx::mbar_arrive_expect_tx(lfull(sl), TB);
                    ptx::tma_load_2d_hint(ptx::smem_u32(lq(sl)), &mq, lfull(sl), 0, row0 + t * kTile, stream_policy);
                    if (early > 0 && t == early - 1 && !(ok = issue_prefix(bh, b, nu))) break;
                }
                ++nu;
            }
            // end marker for the transform warps
            const int sl = k % NL;
            if (ok && (k < NL || ptx::mbar_wait_bounded(lempty(sl), ((k / NL) - 1) & 1, watchdog, WD_OUT_EMPTY,
                                                        kWaitLimitNs))) {
                linfo[8 * sl] = kEndFirst;
                ptx::mbar_arrive(lfull(sl));
            }
        }
    } else if (warp >= 9 * NP) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            for (int k = 0;; ++k) {
                const int so = k % NO, a = k % NA;
                if (flags[0] || !ptx::mbar_wait_bounded(ofull(so), (k / NO) & 1, watchdog, WD_OUT_READY, kWaitLimitNs)) {
                    flags[0] = 1;
                    break;
                }
                const int *inf = oinfo + 8 * so;
                const int u = ld_volatile(inf), ord = ld_volatile(inf + 3), last = ld_volatile(inf + 5);
                if (u < 0) break;
                if (k >= NA &&
                    !ptx::mbar_wait_bounded(acce(a), ((k / NA) - 1) & 1, watchdog, WD_OUT_ACCE, kWaitLimitNs)) {
                    flags[0] = 1;
                    break;
                }
                ptx::tc_fence_after_sync();
                const uint32_t qa = ptx::smem_u32(oq(so)), pa = ptx::smem_u32(oph(so));
                const uint32_t ba = ptx::smem_u32(bbuf + (ord & 1) * C::IMG);
                const uint32_t dacc = tmem + a * C::ACOLS;
#pragma unroll
                for (int kk = 0; kk < 2 * D / 16; ++kk) {
                    // K atom 0 = q~, K atom 1 = phi(q); +32 B per 16-element K step
                    const int atom = kk / (D / 16), j = kk % (D / 16);
                    const uint64_t ad = ptx::smem_desc((atom ? pa : qa) + 32 * j, 16, 8 * ROWB, C::LAYOUT);
                    const uint64_t bd = ptx::smem_desc(ba + atom * C::BATOM + 32 * j, 16, 8 * ROWB, C::LAYOUT);
                    ptx::mma_bf16_ss(dacc, ad, bd, IDESC, kk > 0 ? 1u : 0u);
                }
                ptx::mma_commit(tdone(k % NT));
                if (last) ptx::mma_commit(bempty(ord & 1));
            }
            // every MMA (and the arrivals of the commits above) completes before the CTA's
            // final barrier and TMEM release, also when a wait gave up
            ptx::mma_commit(drain);
            if (!ptx::mbar_wait_bounded(drain, 0, watchdog, WD_OUT_MMA, kWaitLimitNs)) flags[0] = 1;
        }
    } else if (warp < 4 * NP) {
        // ------------------------------------------------------------ transform warps: one row per thread
        const int r = tid & 127;
        const RopeTab tab = load_rope_tab<PT, PY, PX>(g, s_tab, tid, 128 * NP);
        ptx::named_bar_sync(1, 128 * NP);
        const int dx = kTile % g.Wg, dy = (kTile / g.Wg) % g.Hg, dt = kTile / g.HW;
        TokPos tp{0, 0, 0};
        for (int k = 0;; ++k) {
            const int sl = k % NL, so = k % NO;
            if (flags[0] || !ptx::mbar_wait_bounded(lfull(sl), (k / NL) & 1, watchdog, WD_OUT_FULL, kWaitLimitNs)) {
                flags[0] = 1;
                break;
            }
            const int *inf = linfo + 8 * sl;
            const int u = ld_volatile(inf);
            const int t = ld_volatile(inf + 1), valid = ld_volatile(inf + 2), ord = ld_volatile(inf + 3);
            const int tok0 = ld_volatile(inf + 4), last = ld_volatile(inf + 5);
            if (u >= 0 && t == 0) {
                // a new group: build its B operand from the prefix state (the
                // slot's previous group must be done with it)
                const int bs = ord & 1;
                if ((ord >= 2 && !ptx::mbar_wait_bounded(bempty(bs), ((ord >> 1) - 1) & 1, watchdog, WD_OUT_BREADY,
                                                         kWaitLimitNs)) ||
                    !ptx::mbar_wait_bounded(pfull(0), ord & 1, watchdog, WD_OUT_BREADY, kWaitLimitNs)) {
                    flags[0] = 1;
                    break;
                }
                const float *pre = reinterpret_cast<const float *>(pbuf);
                uint4 *dst = reinterpret_cast<uint4 *>(bbuf + bs * C::IMG);
                for (int item = r; item < C::IMG / 16; item += 128) dst[item] = b_operand_chunk<D>(pre, item);
                ptx::fence_proxy_async_smem();  // read by the MMA (async proxy); ordered by this tile's ofull
                warp_arrive(pempty(0), lane);
            }
            uint32_t w[D / 2], ph[D / 2];
            const bool live = u >= 0 && r < valid;
            if (live) load_row<D>(lq(sl), r, w);
            // the next TMA into this slot writes through the async proxy: order
            // this thread's generic reads of the slot before it
            ptx::fence_proxy_async_smem();
            if (u >= 0) warp_arrive(lempty(sl), lane);  // landing slot read
            // operand slot so was last used by tile k - NO: wait for its MMAs
            if (k >= NO && !ptx::mbar_wait_bounded(tdone((k - NO) % NT), ((k - NO) / NT) & 1, watchdog, WD_OUT_READY,
                                                   kWaitLimitNs)) {
                flags[0] = 1;
                break;
            }
            if (u < 0) {  // pass the end on to the MMA issuer, in operand order
                if (r == 0) oinfo[8 * so] = kEndFirst;
                warp_arrive(ofull(so), lane);
                break;
            }
            if (t == 0) tp.init(g, tok0 + r);
            else tp.advance(g, dx, dy, dt);
            if (live) {
                phi_rope_row<D, PT, PY, PX, false>(w, ph, tab, tp, nullptr);
                store_row<D>(oq(so), r, w);
                store_row<D>(oph(so), r, ph);
            } else {  // rows past the group: finite values, outputs not stored
                zero_row<D>(oq(so), r);
                zero_row<D>(oph(so), r);
            }
            ptx::fence_proxy_async_smem();
            if (r == 0) {
                int *oi = oinfo + 8 * so;
                oi[0] = u;
                oi[1] = t;
                oi[3] = ord;
                oi[5] = last;
            }
            warp_arrive(ofull(so), lane);
        }
    } else {
        // ------------------------------------------------------------ epilogue warps: one row per thread
        const int sub = warp & 3, r = 32 * sub + lane;  // tile row = this warp's TMEM subpartition lane
        uint8_t *stg = ostg + sub * 32 * ROWB;           // this warp's 32 staged rows (swizzled like `mo`)
        if (lane == 0) ptx::tma_prefetch_map(&mo);
        const uint64_t stream_policy = ptx::l2_evict_first();  // O is written once
        int k = 0;
        for (int u = u0; u < units && !flags[0]; u += ustep) {  // the producer's tile sequence
            int bh, b, qc;
            decode(u, bh, b, qc);
            const int fb = block_frame_begin(g, b), fe = block_frame_end(g, b);
            const int bntok = (fe - fb) * g.HW, qs = qc * QG;
            if (qs >= bntok) continue;
            const int qlen = min(QG, bntok - qs), ntiles = (qlen + kTile - 1) / kTile;
            const int row0 = bh * g.N + fb * g.HW + qs;
            for (int t = 0; t < ntiles; ++t, ++k) {
                const int a = k % NA;
                if (!ptx::mbar_wait_bounded(tdone(k % NT), (k / NT) & 1, watchdog, WD_OUT_MMA, kWaitLimitNs)) {
                    flags[0] = 1;
                    break;
                }
                ptx::tc_fence_after_sync();
                const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * sub) << 16) + a * C::ACOLS;
                float zh, zl;
                tmem_ld_2cols(taddr + D, zh, zl);
                const float inv = __frcp_rn(zh + zl + g.eps);
                uint32_t ow[D / 2];
#pragma unroll
                for (int half = 0; half < D / 32; ++half) {
                    float v[32];
                    ptx::tmem_ld_32cols(taddr + 32 * half, v);
#pragma unroll
                    for (int q = 0; q < 16; ++q) ow[16 * half + q] = pack_bf16x2(v[2 * q] * inv, v[2 * q + 1] * inv);
                }
                ptx::tc_fence_before_sync();
                warp_arrive(acce(a), lane);  // the accumulator is read: the MMA may overwrite it
                const int valid = min(kTile, qlen - t * kTile);
                if (32 * sub + 32 <= valid) {
                    // whole warp in range: stage the 32 rows and store them with TMA
                    if (lane == 0) ptx::bulk_wait_group_read<0>();  // the previous store has read the staging
                    __syncwarp();
                    store_row<D>(stg, lane, ow);
                    ptx::fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        ptx::tma_store_2d_hint(&mo, ptx::smem_u32(stg), 0, row0 + t * kTile + 32 * sub, stream_policy);
                        ptx::bulk_commit_group();
                    }
                } else if (r < valid) {  // a ragged tile's edge: plain stores of the valid rows
                    uint4 *dst = reinterpret_cast<uint4 *>(o + ((size_t)row0 + t * kTile + r) * D);
#pragma unroll
                    for (int j = 0; j < D / 8; ++j) dst[j] = make_uint4(ow[4 * j], ow[4 * j + 1], ow[4 * j + 2], ow[4 * j + 3]);
                }
            }
        }
        if (lane == 0) ptx::bulk_wait_group<0>();  // stores complete before the CTA exits
    }
    ptx::tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after_sync();
        ptx::tmem_dealloc(*tmem_slot, C::TCOLS);
    }
}

}  // namespace blin
