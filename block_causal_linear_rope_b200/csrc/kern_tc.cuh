// Tensor-core path for bf16 (or NVFP4) Q/K/V on sm_100a (d = 32 or 64): two
// persistent warp-specialized kernels around the fixed-order block scan.
//
// Pass 1, partial_tc_kernel: per state chunk (whole 128-token tiles of one
//   block of one head) the partial states P = sum (R_m phi(k_m)) v_m^T and
//   zp = sum phi(k_m) from one contraction
//       [K~^T ; phi(K)^T] x [V | 1]      (tcgen05.mma, fp32 in TMEM)
//   whose operands are MN-major views of the token-major tiles.
// Pass 2, output_tc_kernel: per group of query tiles of one block of one head,
//   numerator and denominator from one contraction
//       [Q~ | phi(Q)] x [[S, 0], [0, z_hi z_lo]] = [num | phi(q).z_hi | phi(q).z_lo]
//   then o = num / (phi(q).z + eps) in fp32, stored as bf16.
//
// Each CTA (one per SM) runs two pipelines at d = 32, one at d = 64.  A
// pipeline is split into roles -- a TMA producer, four transform warps, one
// MMA-issuing thread, four epilogue warps -- that hand tiles to each other
// through mbarrier rings, and takes its work units one at a time from a
// counter shared by the whole grid.  Every wait is bounded.  With NVFP4 inputs
// the producer lands the packed codes and their block scales, and the
// transform warps decode them (E2M1 x E4M3 products are exact in bf16) before
// phi and RoPE; the global scales are applied in fp32.
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

// A CTA's shared-memory RoPE table: (cos, sin) of every (position, pair) of the
// call's frame window and of every row and column, one section per axis, each
// position-major ([position][pair], the order rope_entry enumerates).  A token row
// reads its position's pairs two at a time (16-byte loads at an offset known at
// compile time from one base per axis); across a warp the t and y entries are
// mostly broadcasts, and consecutive columns sit 48 bytes apart (d = 32), which
// the 16-byte loads of a quarter-warp take without bank conflicts.
struct RopeTab {
    const float4 *t, *y, *x;  // section bases; t indexed by relative frame (window offset folded in)
};

// Fills this CTA's shared-memory RoPE table (the tensor-core path is only
// chosen when it fits; transform threads only, a barrier among them must
// follow).  Entry values are those of rope_entry (same order of operations).
template <int PT, int PY, int PX>
__device__ __forceinline__ RopeTab load_rope_tab(const KGeom &g, float2 *s_tab, int tid, int nthreads) {
    static_assert(PT % 2 == 0 && PY % 2 == 0 && PX % 2 == 0, "pairs are read two at a time");
    const int n = g.T * PT + g.Hg * PY + g.Wg * PX;
    for (int i = tid; i < n; i += nthreads) s_tab[i] = rope_entry(i, g.T, g.t0, g.Hg, PT, PY, PX, g.theta);
    RopeTab r;
    r.t = reinterpret_cast<const float4 *>(s_tab);
    r.y = reinterpret_cast<const float4 *>(s_tab + g.tab_y);
    r.x = reinterpret_cast<const float4 *>(s_tab + g.tab_x);
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
    const float4 *rt = tab.t + tp.t * (PT / 2);
    const float4 *ry = tab.y + tp.y * (PY / 2);
    const float4 *rx = tab.x + tp.x * (PX / 2);
#pragma unroll
    for (int q = 0; q < D / 4; ++q) {  // pairs 2q, 2q + 1 (never straddling two axes)
        const int p0 = 2 * q;
        const float4 cs2 = p0 < PT ? rt[q] : (p0 < PT + PY ? ry[q - PT / 2] : rx[q - (PT + PY) / 2]);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int p = p0 + h;
            const float c = h ? cs2.z : cs2.x, sn = h ? cs2.w : cs2.y;
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
            w[p] = pack_bf16x2(fmaf(a, c, -b * sn), fmaf(a, sn, b * c));
        }
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

// ============================================================================ work units
// Unit r of a head (pass-1 chunks or pass-2 query groups, ordered by block):
// block b and index c inside the block.
__device__ __forceinline__ void unit_block(const KGeom &g, int r, int nf, int nm, int nl, int &b, int &c) {
    if (r < nf) {
        b = 0;
        c = r;
        return;
    }
    r -= nf;
    const int mids = g.nblk > 2 ? g.nblk - 2 : 0;
    if (r < mids * nm) {
        b = 1 + r / nm;
        c = r - (b - 1) * nm;
        return;
    }
    b = g.nblk - 1;
    c = r - mids * nm;
}

// 4D tensor-map coordinates (feature, token, head, batch) in the map's own
// dimension order: dims 1 and 2 are ordered by stride, so `swap` puts the head
// before the token (a token-interleaved [B][N][H][d] layout).
struct MapCoord {
    int y, z;
};
__device__ __forceinline__ MapCoord map_coord(int n, int h, int swap) { return swap ? MapCoord{h, n} : MapCoord{n, h}; }

// ============================================================================ configuration
template <int D>
struct TcCfg {
    static constexpr int ROWB = 2 * D;
    static constexpr int TB = kTile * ROWB;           // one 128-token tile: 8 KB (d = 32) / 16 KB (d = 64)
    static constexpr int NP = D == 32 ? 2 : 1;        // pipelines per CTA
    static constexpr int PIPE_WARPS = 10;             // per pipeline: 4 transform, 4 epilogue, producer, MMA
    static constexpr int THREADS = 32 * PIPE_WARPS * NP;
    static constexpr uint32_t LAYOUT = D == 32 ? 4u : 2u;  // smem descriptor swizzle: 64B / 128B
    static constexpr int ACOLS = D == 32 ? 64 : 128;       // TMEM columns per accumulator
    static constexpr int NINFO = 16;                        // producer -> epilogue record ring
    static constexpr int NO = 2;                            // operand slots
    static constexpr int NA = 4;                            // TMEM accumulators per pipeline
    static constexpr uint32_t TCOLS = 512;
    static constexpr int E = D * D + D, E4 = E / 4;
    // control block: [NP][BARS_PER_PIPE] mbarriers, 16 B of flags, [NP][INFO_PER_PIPE] record ints
    static constexpr int BARS_PER_PIPE = 72;
    static constexpr int INFO_PER_PIPE = 160;
    static constexpr int OFF_FLAGS = NP * BARS_PER_PIPE * 8;
    static constexpr int OFF_INFO = OFF_FLAGS + 16;
    static constexpr int CTRL = (OFF_INFO + NP * INFO_PER_PIPE * 4 + 1023) / 1024 * 1024;
    static_assert(NP * NA * ACOLS <= (int)TCOLS, "TMEM columns");
};

// NVFP4 inputs (FP4 = true): a tile of 128 tokens is d/2 packed bytes per token
// (two E2M1 codes a byte) and d/16 E4M3 scale bytes per token.
template <int D>
struct Fp4Tile {
    static constexpr int DB = D / 2 * kTile;        // packed data bytes of one tile
    static constexpr int S1 = D / 16;               // scale bytes per token
    static constexpr int SB = S1 * kTile + 32;      // scale bytes of one tile, with room to round the copy to 16 B
    static constexpr int TABS = 256 * 4 + 256 * 2;  // dequantisation tables: code pairs, E4M3 scales
};

template <int D, bool FP4 = false>
struct K1Cfg : TcCfg<D> {
    using B = TcCfg<D>;
    using F = Fp4Tile<D>;
    static constexpr int M1 = D == 32 ? 64 : 128;          // [K~^T ; phi(K)^T]
    static constexpr int N1 = D == 32 ? D + 8 : D + 16;    // [V | ones]
    // landing slots: bf16 -- one K tile (free once read); NVFP4 -- a tile's K and V data
    // and scales (free once read: V is dequantised into the operand slot)
    static constexpr int LSLOT = FP4 ? (2 * (F::DB + F::SB) + 1023) / 1024 * 1024 : B::TB;
    static constexpr int NK = FP4 ? (D == 32 ? 8 : 6) : (D == 32 ? 4 : 3);
    static constexpr int NV = FP4 ? 0 : 4;                 // bf16 V landing slots (read in place by the MMA)
    static constexpr int NTD = FP4 ? 4 : NV;               // tile-done barriers
    static constexpr int OPND = (FP4 ? 3 : 2) * B::TB;     // operand slot: K~ | phi (| dequantised V)
    static constexpr int PIPE = NK * LSLOT + NV * B::TB + B::NO * OPND;
    static constexpr int OFF_ONES = B::NP * PIPE;          // above every V tile: positive LBO
    static constexpr int OFF_CTRL = OFF_ONES + B::TB;
    static constexpr int TABS = FP4 ? F::TABS : 0;         // after the control block
    static constexpr int FIXED = OFF_CTRL + B::CTRL + TABS + 1024;  // + alignment slack; the RoPE table follows
    static constexpr int LREC = 7;                         // ints per landing record
    static constexpr int NBAR = 2 * NK + NTD + B::NO + 2 * B::NA + 2 * B::NINFO + 1;
    static constexpr int NINF = LREC * NK + 4 * B::NO + B::NINFO;
    static_assert(NBAR <= B::BARS_PER_PIPE && NINF <= B::INFO_PER_PIPE, "control block");
    static_assert(NTD > B::NO, "an operand slot's release is read from the tile-done barriers");
    static_assert(OFF_ONES < (1 << 18), "LBO field range");
    static_assert(PIPE % 1024 == 0, "pipelines keep 1024-byte alignment");
};

template <int D, bool FP4 = false>
struct K2Cfg : TcCfg<D> {
    using B = TcCfg<D>;
    using F = Fp4Tile<D>;
    // Q lands one tile per slot (bf16: one TMA box; NVFP4: a tile's data and scales)
    static constexpr int SPAN = 1;                             // tiles per Q landing slot
    static constexpr int NLS = FP4 ? 8 : (D == 32 ? 5 : 3);    // Q landing slots
    static constexpr int LSLOT = FP4 ? (F::DB + F::SB + 1023) / 1024 * 1024 : SPAN * B::TB;
    static constexpr int NL = NLS * SPAN;                      // Q tiles in the landing ring
    static constexpr int NT = B::NA > B::NO + 1 ? B::NA : B::NO + 1;  // tile-done barriers
    static constexpr int N2 = OutB<D>::N;
    static constexpr int BATOM = OutB<D>::BATOM;
    static constexpr int IMG = OutB<D>::IMG;
    static constexpr int PRE = (D * D + D) * 4;            // one fp32 prefix state (S, z)
    // Q ring, operand ring, O staging (4 warps x 32 rows), 2 B images, 2 prefix states
    // (a group's prefix is fetched while the previous group is still being computed)
    static constexpr int PIPE = (NLS * LSLOT + B::NO * 2 * B::TB + B::TB + 2 * IMG + 2 * PRE + 1023) / 1024 * 1024;
    static constexpr int OFF_CTRL = B::NP * PIPE;
    static constexpr int TABS = FP4 ? F::TABS : 0;
    static constexpr int FIXED = OFF_CTRL + B::CTRL + TABS + 1024;
    static constexpr int NBAR = 2 * NLS + B::NO + NT + B::NA + 6 + 2 * B::NINFO + 1;
    static constexpr int NINF = 8 * NLS + 6 * B::NO + 4 * B::NINFO;
    static_assert(NBAR <= B::BARS_PER_PIPE && NINF <= B::INFO_PER_PIPE, "control block");
};

// ---------------------------------------------------------------------------- NVFP4 decoding
// Tables in shared memory, filled once per CTA: pair[byte] = the two E2M1 values of a
// packed byte as bf16x2 (even element in the low half); e4m3[byte] = the E4M3 scale as
// bf16 bits.  Every E2M1 x E4M3 product has at most 6 significant bits, so multiplying
// the bf16 pair by the bf16 scale is exact: the tile's bf16 values are exactly the
// NVFP4 values up to the tensor's global scale (applied in fp32 by the epilogues).
__device__ __forceinline__ float e2m1_value(int c) {
    const int e = (c >> 1) & 3, m = c & 1;
    const float mag = e == 0 ? 0.5f * m : ldexpf(1.0f + 0.5f * m, e - 1);
    return (c & 8) ? -mag : mag;
}
__device__ __forceinline__ float e4m3_value(int c) {
    const int e = (c >> 3) & 15, m = c & 7;
    const float mag = e == 0 ? ldexpf(m / 8.0f, -6) : ldexpf(1.0f + m / 8.0f, e - 7);
    return (c & 0x80) ? -mag : mag;  // codes 0x7f / 0xff (NaN) are never produced by a valid encoder
}
__device__ __forceinline__ void fill_fp4_tables(uint8_t *tabs, int tid, int nthreads) {
    uint32_t *pair = reinterpret_cast<uint32_t *>(tabs);
    uint16_t *sc = reinterpret_cast<uint16_t *>(tabs + 1024);
    for (int i = tid; i < 256; i += nthreads) {
        pair[i] = pack_bf16x2(e2m1_value(i & 15), e2m1_value(i >> 4));
        const __nv_bfloat16 h = __float2bfloat16_rn(e4m3_value(i));
        sc[i] = *reinterpret_cast<const uint16_t *>(&h);
    }
}
// One token row: d/2 packed bytes at `data`, d/16 scale bytes at `scale` -> bf16x2 words.
template <int D>
__device__ __forceinline__ void fp4_row(const uint8_t *data, const uint8_t *scale, const uint8_t *tabs,
                                        uint32_t (&w)[D / 2]) {
    const uint32_t *pair = reinterpret_cast<const uint32_t *>(tabs);
    const uint16_t *sc = reinterpret_cast<const uint16_t *>(tabs + 1024);
#pragma unroll
    for (int j = 0; j < D / 32; ++j) {  // 16 bytes = 32 elements = two scale blocks
        const uint4 v = *reinterpret_cast<const uint4 *>(data + 16 * j);
        const uint32_t words[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const uint32_t sbits = sc[scale[2 * j + half]];
            const uint32_t s2 = sbits | (sbits << 16);
            const __nv_bfloat162 s2h = *reinterpret_cast<const __nv_bfloat162 *>(&s2);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int byte_i = 8 * half + q;
                const uint32_t byte = (words[byte_i >> 2] >> (8 * (byte_i & 3))) & 0xFFu;
                const uint32_t pv = pair[byte];
                const __nv_bfloat162 prod = __hmul2(*reinterpret_cast<const __nv_bfloat162 *>(&pv), s2h);
                w[16 * j + byte_i] = *reinterpret_cast<const uint32_t *>(&prod);
            }
        }
    }
}
// Bytes [a0, a1) of a tile's scale rows: `rows` tokens from global token row `row0`
// (of `total` rows), rounded outwards to 16 bytes (the allocation is padded to 16 B).
struct ScaleSpan {
    long long a0;
    int bytes, off;
};
template <int D>
__device__ __forceinline__ ScaleSpan scale_span(long long row0, int rows, long long total) {
    constexpr int S1 = D / 16;
    const long long b0 = row0 * S1, e = min(row0 + rows, total) * S1;
    ScaleSpan sp;
    sp.a0 = b0 & ~15LL;
    sp.bytes = (int)(((e + 15) & ~15LL) - sp.a0);
    sp.off = (int)(b0 - sp.a0);
    return sp;
}

// Named barrier of all transform warps of a CTA (the RoPE table fill, before
// any work starts; every other hand-over is an mbarrier with a bounded wait).
constexpr uint32_t kBarTab = 4;

// One pipeline's view of shared memory.
struct PipeSmem {
    uint8_t *base;        // the pipeline's rings
    uint64_t *bars;       // its mbarriers
    int *info;            // its records
    volatile int *flags;  // the CTA's: [0] abort
    uint8_t *ones;        // pass 1: constant B block (all 1.0)
};

// ---------------------------------------------------------------------------- pass-1 pipeline
template <int D, int PT, int PY, int PX, bool FP4>
struct Pass1 {
    using C = K1Cfg<D, FP4>;
    using F = Fp4Tile<D>;
    static constexpr int NK = C::NK, NV = C::NV, NTD = C::NTD, NO = C::NO, NA = C::NA, TB = C::TB, ROWB = C::ROWB,
                         E = C::E, LREC = C::LREC;
    static constexpr int NVD = NV > 0 ? NV : 1;  // divisor for the bf16 V ring (unused with NVFP4)
    const KGeom &g;
    PipeSmem ps;
    int *wd;
    uint8_t *kring, *vring, *opnd;
    const uint8_t *tabs;  // NVFP4 decoding tables
    int *linfo, *oinfo, *cinfo;
    uint32_t tmem;

    __device__ Pass1(const KGeom &g_, const PipeSmem &ps_, int *wd_, uint32_t tmem_base, const uint8_t *tabs_)
        : g(g_), ps(ps_), wd(wd_), tabs(tabs_) {
        kring = ps.base;
        vring = kring + NK * C::LSLOT;
        opnd = vring + NV * TB;
        linfo = ps.info;
        oinfo = linfo + LREC * NK;
        cinfo = oinfo + 4 * NO;
        tmem = tmem_base;
    }
    __device__ uint8_t *lk(int s) const { return kring + s * C::LSLOT; }
    __device__ uint8_t *lv(int s) const { return vring + s * TB; }
    __device__ uint8_t *ok_(int s) const { return opnd + s * C::OPND; }
    __device__ uint8_t *op_(int s) const { return opnd + s * C::OPND + TB; }
    __device__ uint8_t *ov_(int s) const { return opnd + s * C::OPND + 2 * TB; }  // NVFP4: dequantised V
    // kfull[s]: the tile in landing slot s has landed (bf16: K, and V in its V slot; NVFP4:
    // K and V data and scales); kempty[s]: slot s is read (4 warps); tdone[s]: the tile
    // k = s (mod NTD) is multiplied (its operand slot, and bf16 V slot, are free);
    // ofull[s]: operand slot s written (4 warps); accf/acce: chunk accumulator ready / read;
    // cfull/cempty: chunk record ring (producer -> epilogue)
    __device__ uint32_t bar(int i) const { return ptx::smem_u32(ps.bars + i); }
    __device__ uint32_t kfull(int s) const { return bar(s); }
    __device__ uint32_t kempty(int s) const { return bar(NK + s); }
    __device__ uint32_t tdone(int s) const { return bar(2 * NK + s); }
    __device__ uint32_t ofull(int s) const { return bar(2 * NK + NTD + s); }
    __device__ uint32_t accf(int a) const { return bar(2 * NK + NTD + NO + a); }
    __device__ uint32_t acce(int a) const { return bar(2 * NK + NTD + NO + NA + a); }
    __device__ uint32_t cfull(int i) const { return bar(2 * NK + NTD + NO + 2 * NA + i); }
    __device__ uint32_t cempty(int i) const { return bar(2 * NK + NTD + NO + 2 * NA + C::NINFO + i); }
    __device__ uint32_t drain() const { return bar(2 * NK + NTD + NO + 2 * NA + 2 * C::NINFO); }

    __device__ static void init_barriers(uint64_t *b) {
        auto at = [&](int i) { return ptx::smem_u32(b + i); };
        for (int s = 0; s < NK; ++s) {
            ptx::mbar_init(at(s), 1);       // kfull: producer (+ TMA bytes)
            ptx::mbar_init(at(NK + s), 4);  // kempty: transform warps
        }
        for (int s = 0; s < NTD; ++s) ptx::mbar_init(at(2 * NK + s), 1);       // tdone: commit
        for (int s = 0; s < NO; ++s) ptx::mbar_init(at(2 * NK + NTD + s), 4);  // ofull
        for (int a = 0; a < NA; ++a) {
            ptx::mbar_init(at(2 * NK + NTD + NO + a), 1);       // accf: commit
            ptx::mbar_init(at(2 * NK + NTD + NO + NA + a), 4);  // acce: epilogue warps
        }
        for (int i = 0; i < C::NINFO; ++i) {
            ptx::mbar_init(at(2 * NK + NTD + NO + 2 * NA + i), 1);            // cfull: producer
            ptx::mbar_init(at(2 * NK + NTD + NO + 2 * NA + C::NINFO + i), 4);  // cempty: epilogue
        }
        ptx::mbar_init(at(2 * NK + NTD + NO + 2 * NA + 2 * C::NINFO), 1);  // drain
    }

    __device__ int nc_of(int b) const { return units_of_block(g, b, g.nc_first, g.nc_mid, g.nc_last); }
    __device__ void decode(int u, int &bh, int &b, int &c) const {
        bh = u / g.U1;
        unit_block(g, u - bh * g.U1, g.nc_first, g.nc_mid, g.nc_last, b, c);
    }

    // ------------------------------------------------------------ TMA producer (lanes 0 and 1)
    // Lane 0 claims chunks, keeps the rings and issues the K loads; lane 1 issues the V
    // loads of the same tiles.  One thread can keep only so many tile loads moving, so
    // two issuing threads move twice the bytes.
    __device__ void producer(const CUtensorMap *mk, const CUtensorMap *mv, int lane) {
        const bool lead = lane == 0;
        if (lead) ptx::tma_prefetch_map(mk);
        else ptx::tma_prefetch_map(mv);
        const uint64_t policy = ptx::l2_evict_first();  // K and V are read once
        const int total = g.BH * g.U1;
        int k = 0, j = 0;
        bool ok = true;
        // claims one ahead, so the atomic's latency is hidden
        int next = lead ? static_cast<int>(atomicAdd(&g.ctl[0], 1u)) : 0;
        next = __shfl_sync(3u, next, 0);
        while (ok && next < total) {
            const int u = next;
            const int nx = lead ? static_cast<int>(atomicAdd(&g.ctl[0], 1u)) : 0;
            next = __shfl_sync(3u, nx, 0);
            int bh, b, c;
            decode(u, bh, b, c);
            const int fb = block_frame_begin(g, b), fe = block_frame_end(g, b);
            const int L = (fe - fb) * g.HW, nt = (L + kTile - 1) / kTile, nc = nc_of(b);
            const int t_lo = c * nt / nc, t_hi = (c + 1) * nt / nc;
            const int bb = bh / g.H, hh = bh - bb * g.H;
            // the chunk's record for the epilogue
            if (lead) {
                const int ci = j % C::NINFO;
                if (j >= C::NINFO &&
                    !ptx::mbar_wait_bounded(cempty(ci), ((j / C::NINFO) - 1) & 1, wd, WD_P1_INFO, kWaitLimitNs)) {
                    ok = false;
                } else {
                    cinfo[ci] = u;
                    ptx::mbar_arrive(cfull(ci));
                }
            }
            ok = __shfl_sync(3u, ok ? 1 : 0, 0) != 0;
            if (!ok) break;
            ++j;
            for (int t = t_lo; t < t_hi; ++t, ++k) {
                const int sk = k % NK, sv = k % NVD;
                const int n = fb * g.HW + t * kTile;  // token (within the head) of the tile's first row
                // NVFP4: this tile's scale bytes, rounded outwards to 16 B (same for K and V)
                ScaleSpan sp{};
                if constexpr (FP4) sp = scale_span<D>((long long)bh * g.N + n, kTile, (long long)g.BH * g.N);
                if (lead) {
                    if ((k >= NK && !ptx::mbar_wait_bounded(kempty(sk), ((k / NK) - 1) & 1, wd, WD_P1_EMPTY, kWaitLimitNs)) ||
                        (!FP4 && k >= NV &&
                         !ptx::mbar_wait_bounded(tdone(sv), ((k / NVD) - 1) & 1, wd, WD_P1_EMPTY, kWaitLimitNs))) {
                        ok = false;
                    } else {
                        int *inf = linfo + LREC * sk;
                        inf[0] = u;
                        inf[1] = t - t_lo;
                        inf[2] = min(kTile, L - t * kTile);
                        inf[3] = t == t_hi - 1;
                        inf[4] = n;
                        inf[5] = sp.off;
                        ptx::mbar_arrive_expect_tx(kfull(sk), FP4 ? 2 * (F::DB + sp.bytes) : 2 * TB);
                    }
                }
                // both slots are free (and the bytes expected) before either load goes out
                ok = __shfl_sync(3u, ok ? 1 : 0, 0) != 0;
                if (!ok) break;
                const MapCoord mc = map_coord(n, hh, g.swap_q);
                if constexpr (FP4) {
                    // lane 0: K data and scales; lane 1: V data and scales
                    uint8_t *slot = lk(sk);
                    const uint8_t *sg = lead ? g.sk_scale : g.sv_scale;
                    ptx::tma_load_4d_hint(ptx::smem_u32(slot + (lead ? 0 : F::DB)), lead ? mk : mv, kfull(sk), 0, mc.y,
                                          mc.z, bb, policy);
                    ptx::bulk_load(ptx::smem_u32(slot + 2 * F::DB + (lead ? 0 : F::SB)), sg + sp.a0, sp.bytes, kfull(sk));
                } else {
                    if (lead) ptx::tma_load_4d_hint(ptx::smem_u32(lk(sk)), mk, kfull(sk), 0, mc.y, mc.z, bb, policy);
                    else ptx::tma_load_4d_hint(ptx::smem_u32(lv(sv)), mv, kfull(sk), 0, mc.y, mc.z, bb, policy);
                }
            }
        }
        if (!lead) return;
        // end markers: transform warps (through the landing ring) and epilogue (chunk ring)
        const int sk = k % NK;
        bool marked = false;
        if (ok && (k < NK || ptx::mbar_wait_bounded(kempty(sk), ((k / NK) - 1) & 1, wd, WD_P1_EMPTY, kWaitLimitNs))) {
            linfo[LREC * sk] = kEndFirst;
            ptx::mbar_arrive(kfull(sk));
            marked = true;
        }
        const int ci = j % C::NINFO;
        if (ok && (j < C::NINFO ||
                   ptx::mbar_wait_bounded(cempty(ci), ((j / C::NINFO) - 1) & 1, wd, WD_P1_INFO, kWaitLimitNs))) {
            cinfo[ci] = kEndFirst;
            ptx::mbar_arrive(cfull(ci));
        }
        // No TMA write may still be in flight into this CTA's shared memory when it exits.
        // Tiles before k - NK were seen landed before their slots were refilled; tile k - NK
        // too when the end marker went into its slot (that waited for the slot's release).
        // The end marker moved that slot's phase on, so it must not be waited for again.
        // (kfull counts the V bytes too.)
        const int oldest = marked ? k - NK + 1 : k - NK;
        for (int kk = k - 1; kk >= 0 && kk >= oldest; --kk)
            ptx::mbar_wait_bounded(kfull(kk % NK), (kk / NK) & 1, wd, WD_P1_FULL, kWaitLimitNs);
    }

    // ------------------------------------------------------------ MMA issuer (one thread)
    __device__ void mma() {
        constexpr uint32_t IDESC = ptx::idesc_bf16_f32(C::M1, C::N1, 1, 1);
        int nu = 0;
        for (int k = 0;; ++k) {
            const int so = k % NO;
            if (ps.flags[0] || !ptx::mbar_wait_bounded(ofull(so), (k / NO) & 1, wd, WD_P1_READY, kWaitLimitNs)) {
                ps.flags[0] = 1;
                break;
            }
            const int *inf = oinfo + 4 * so;
            const int u = ld_volatile(inf), t = ld_volatile(inf + 1), last = ld_volatile(inf + 3);
            if (u < 0) break;
            const int a = nu % NA;
            if (t == 0 && nu >= NA &&
                !ptx::mbar_wait_bounded(acce(a), ((nu / NA) - 1) & 1, wd, WD_P1_ACC, kWaitLimitNs)) {
                ps.flags[0] = 1;
                break;
            }
            ptx::tc_fence_after_sync();
            // the tile's V: bf16 in place in its landing slot; NVFP4 dequantised in the operand slot
            const uint32_t va = FP4 ? ptx::smem_u32(ov_(so)) : ptx::smem_u32(lv(k % NVD));
            // A (MN-major): M atom 0 = K~ rows, atom 1 (+TB) = phi rows; B: V | ones.
            // Consecutive K steps are 16 token rows (16 * ROWB bytes: ROWB in the address field).
            const uint64_t ad = ptx::smem_desc(ptx::smem_u32(ok_(so)), TB, 8 * ROWB, C::LAYOUT);
            const uint64_t bd = ptx::smem_desc(va, ptx::smem_u32(ps.ones) - va, 8 * ROWB, C::LAYOUT);
            const uint32_t dacc = tmem + a * C::ACOLS;
#pragma unroll
            for (int kk = 0; kk < kTile / 16; ++kk)
                ptx::mma_bf16_ss(dacc, ad + static_cast<uint64_t>(kk * ROWB), bd + static_cast<uint64_t>(kk * ROWB),
                                 IDESC, (t > 0 || kk > 0) ? 1u : 0u);
            ptx::mma_commit(tdone(k % NTD));
            if (last) {
                ptx::mma_commit(accf(a));
                ++nu;
            }
        }
        // every MMA (and the arrivals of the commits above) completes before the CTA's
        // final barrier and TMEM release, also when a wait gave up
        ptx::mma_commit(drain());
        if (!ptx::mbar_wait_bounded(drain(), 0, wd, WD_P1_DRAIN, kWaitLimitNs)) ps.flags[0] = 1;
    }

    // ------------------------------------------------------------ transform warps (one row per thread)
    __device__ void transform(const RopeTab &tab, int r) {
        const int lane = r & 31;
        const int dx = kTile % g.Wg, dy = (kTile / g.Wg) % g.Hg, dt = kTile / g.HW;
        TokPos tp{0, 0, 0};
        for (int k = 0;; ++k) {
            const int sk = k % NK, so = k % NO;
            if (ps.flags[0] || !ptx::mbar_wait_bounded(kfull(sk), (k / NK) & 1, wd, WD_P1_FULL, kWaitLimitNs)) {
                ps.flags[0] = 1;
                break;
            }
            const int *inf = linfo + LREC * sk;
            const int u = ld_volatile(inf), t = ld_volatile(inf + 1), valid = ld_volatile(inf + 2);
            const int last = ld_volatile(inf + 3), n = ld_volatile(inf + 4);
            // read this row of K; rows past the chunk also clear their V row
            // (the MMA reads V in place: other blocks' tokens must add nothing)
            uint32_t w[D / 2], ph[D / 2], vw[D / 2];
            const bool live = u >= 0 && r < valid;
            if constexpr (FP4) {
                if (live) {
                    const uint8_t *slot = lk(sk), *scl = slot + 2 * F::DB + ld_volatile(inf + 5) + r * F::S1;
                    fp4_row<D>(slot + r * (D / 2), scl, tabs, w);
                    fp4_row<D>(slot + F::DB + r * (D / 2), scl + F::SB, tabs, vw);
                }
            } else {
                if (live) load_row<D>(lk(sk), r, w);
                else if (u >= 0) zero_row<D>(lv(k % NVD), r);
            }
            // the next TMA into this K slot writes through the async proxy: order
            // this thread's generic reads of the slot before it
            ptx::fence_proxy_async_smem();
            if (u >= 0) warp_arrive(kempty(sk), lane);
            // operand slot so was last used by tile k - NO: wait for its MMAs
            if (k >= NO && !ptx::mbar_wait_bounded(tdone((k - NO) % NTD), ((k - NO) / NTD) & 1, wd, WD_P1_READY,
                                                   kWaitLimitNs)) {
                ps.flags[0] = 1;
                break;
            }
            if (u < 0) {  // pass the end on to the MMA issuer, in operand order
                if (r == 0) oinfo[4 * so] = kEndFirst;
                warp_arrive(ofull(so), lane);
                break;
            }
            if (t == 0) tp.init(g, n + r);
            else tp.advance(g, dx, dy, dt);
            if (live) {
                phi_rope_row<D, PT, PY, PX, false>(w, ph, tab, tp, nullptr);
                store_row<D>(ok_(so), r, w);
                store_row<D>(op_(so), r, ph);
                if constexpr (FP4) store_row<D>(ov_(so), r, vw);
            } else {  // rows past the chunk add nothing
                zero_row<D>(ok_(so), r);
                zero_row<D>(op_(so), r);
                if constexpr (FP4) zero_row<D>(ov_(so), r);
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
        }
    }

    // ------------------------------------------------------------ epilogue warps: chunk partials
    // `e` is the thread's index in the 4 epilogue warps; `sub` its warp's TMEM subpartition.
    __device__ void epilogue(int e, int sub) {
        const int lane = e & 31;
        constexpr int RPS = D == 32 ? 16 : 32;  // accumulator rows per TMEM subpartition
        for (int j = 0;; ++j) {
            const int ci = j % C::NINFO;
            if (ps.flags[0] || !ptx::mbar_wait_bounded(cfull(ci), (j / C::NINFO) & 1, wd, WD_P1_INFO, kWaitLimitNs)) {
                ps.flags[0] = 1;
                break;
            }
            const int u = ld_volatile(cinfo + ci);
            warp_arrive(cempty(ci), lane);
            if (u < 0) break;
            const int a = j % NA;
            if (!ptx::mbar_wait_bounded(accf(a), (j / NA) & 1, wd, WD_P1_ACC, kWaitLimitNs)) {
                ps.flags[0] = 1;
                break;
            }
            ptx::tc_fence_after_sync();
            int bh, b, c;
            decode(u, bh, b, c);
            float *out = g.part + (((size_t)bh * g.nblk + b) * g.cpb + c) * E;
            // M = 64 (d = 32): accumulator row m in TMEM lane (m % 16) + 32 * (m / 16);
            // M = 128 (d = 64): row m in lane m.  Rows [0, D) hold P, rows [D, 2D) hold
            // phi^T against the ones block, i.e. zp, in column D.
            const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * sub) << 16) + a * C::ACOLS;
            if (sub < 2) {
                const int m = RPS * sub + lane;  // P row
                const float sp = FP4 ? g.gk * g.gv : 1.0f;  // NVFP4: the tensors' global scales
#pragma unroll
                for (int half = 0; half < D / 32; ++half) {
                    float v[32];
                    ptx::tmem_ld_32cols(taddr + 32 * half, v);
                    if constexpr (FP4) {
#pragma unroll
                        for (int q = 0; q < 32; ++q) v[q] *= sp;
                    }
                    if (lane < RPS) {
                        float4 *dst = reinterpret_cast<float4 *>(out + m * D + 32 * half);
#pragma unroll
                        for (int q = 0; q < 8; ++q) dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                    }
                }
            } else {
                float zv, unused;
                tmem_ld_2cols(taddr + D, zv, unused);
                if constexpr (FP4) zv *= g.gk;
                if (lane < RPS) out[D * D + RPS * (sub - 2) + lane] = zv;
            }
            ptx::tc_fence_before_sync();
            warp_arrive(acce(a), lane);  // accumulator a is free again
        }
    }
};

// ---------------------------------------------------------------------------- pass-2 pipeline
template <int D, int PT, int PY, int PX, bool FP4>
struct Pass2 {
    using C = K2Cfg<D, FP4>;
    using F = Fp4Tile<D>;
    static constexpr int NL = C::NL, NLS = C::NLS, SPAN = C::SPAN, NO = C::NO, NA = C::NA, NT = C::NT, TB = C::TB,
                         ROWB = C::ROWB, E = C::E;
    const KGeom &g;
    PipeSmem ps;
    int *wd;
    uint8_t *land, *opnd, *ostg, *bbuf, *pbuf;
    const uint8_t *tabs;  // NVFP4 decoding tables
    int *linfo, *oinfo, *tinfo;
    uint32_t tmem;

    __device__ Pass2(const KGeom &g_, const PipeSmem &ps_, int *wd_, uint32_t tmem_base, const uint8_t *tabs_)
        : g(g_), ps(ps_), wd(wd_), tabs(tabs_) {
        land = ps.base;
        opnd = land + NLS * C::LSLOT;
        ostg = opnd + NO * 2 * TB;
        bbuf = ostg + TB;
        pbuf = bbuf + 2 * C::IMG;
        linfo = ps.info;
        oinfo = linfo + 8 * NLS;
        tinfo = oinfo + 6 * NO;
        tmem = tmem_base;
    }
    __device__ uint8_t *lq(int s) const { return land + s * C::LSLOT; }
    __device__ uint8_t *oq(int s) const { return opnd + s * 2 * TB; }
    __device__ uint8_t *oph(int s) const { return opnd + s * 2 * TB + TB; }
    __device__ uint32_t bar(int i) const { return ptx::smem_u32(ps.bars + i); }
    __device__ uint32_t lfull(int s) const { return bar(s); }
    __device__ uint32_t lempty(int s) const { return bar(NLS + s); }
    __device__ uint32_t ofull(int s) const { return bar(2 * NLS + s); }
    __device__ uint32_t tdone(int s) const { return bar(2 * NLS + NO + s); }
    __device__ uint32_t acce(int a) const { return bar(2 * NLS + NO + NT + a); }
    // pfull[s] / pempty[s]: prefix buffer s landed / turned into a B image (4 warps)
    __device__ uint32_t pfull(int s) const { return bar(2 * NLS + NO + NT + NA + s); }
    __device__ uint32_t pempty(int s) const { return bar(2 * NLS + NO + NT + NA + 2 + s); }
    __device__ uint32_t bempty(int s) const { return bar(2 * NLS + NO + NT + NA + 4 + s); }
    __device__ uint32_t tfull(int i) const { return bar(2 * NLS + NO + NT + NA + 6 + i); }
    __device__ uint32_t tempty(int i) const { return bar(2 * NLS + NO + NT + NA + 6 + C::NINFO + i); }
    __device__ uint32_t drain() const { return bar(2 * NLS + NO + NT + NA + 6 + 2 * C::NINFO); }
    __device__ uint8_t *prefix_buf(int s) const { return pbuf + s * C::PRE; }

    __device__ static void init_barriers(uint64_t *b) {
        auto at = [&](int i) { return ptx::smem_u32(b + i); };
        for (int s = 0; s < NLS; ++s) {
            ptx::mbar_init(at(s), 1);        // lfull: producer + TMA bytes
            ptx::mbar_init(at(NLS + s), 4);  // lempty: transform warps
        }
        for (int s = 0; s < NO; ++s) ptx::mbar_init(at(2 * NLS + s), 4);           // ofull
        for (int s = 0; s < NT; ++s) ptx::mbar_init(at(2 * NLS + NO + s), 1);      // tdone: commit
        for (int a = 0; a < NA; ++a) ptx::mbar_init(at(2 * NLS + NO + NT + a), 4);  // acce: epilogue
        for (int s = 0; s < 2; ++s) {
            ptx::mbar_init(at(2 * NLS + NO + NT + NA + s), 1);      // pfull: bulk copy
            ptx::mbar_init(at(2 * NLS + NO + NT + NA + 2 + s), 4);  // pempty: transform
            ptx::mbar_init(at(2 * NLS + NO + NT + NA + 4 + s), 1);  // bempty: commit
        }
        for (int i = 0; i < C::NINFO; ++i) {
            ptx::mbar_init(at(2 * NLS + NO + NT + NA + 6 + i), 1);              // tfull: producer
            ptx::mbar_init(at(2 * NLS + NO + NT + NA + 6 + C::NINFO + i), 4);  // tempty: epilogue
        }
        ptx::mbar_init(at(2 * NLS + NO + NT + NA + 6 + 2 * C::NINFO), 1);  // drain
    }

    __device__ int ng_of(int b) const { return units_of_block(g, b, g.ng_first, g.ng_mid, g.ng_last); }

    // ------------------------------------------------------------ producer (one thread)
    // Q goes out in spans of SPAN tiles of one group, one TMA box (SPAN * 128 rows) per
    // landing slot; rows past the group's block are masked by the transform warps.
    __device__ void producer(const CUtensorMap *mq) {
        ptx::tma_prefetch_map(mq);
        const uint64_t policy = ptx::l2_evict_first();  // Q is read once
        const int total = g.BH * g.U2;
        int kp = 0, j = 0, nu = 0, npre = 0;
        bool ok = true, waited = false;
        // group nu's fp32 prefix state (written by the block scan, the previous kernel) into
        // buffer nu & 1, as soon as group nu - 2 has turned that buffer into its B image
        auto issue_prefix = [&](int bh, int b) {
            const int ps_ = nu & 1;
            if (nu >= 2 && !ptx::mbar_wait_bounded(pempty(ps_), ((nu >> 1) - 1) & 1, wd, WD_P2_BREADY, kWaitLimitNs))
                return false;
            if (!waited) {
                griddep_wait();
                waited = true;
            }
            ptx::mbar_arrive_expect_tx(pfull(ps_), C::PRE);
            ptx::bulk_load(ptx::smem_u32(prefix_buf(ps_)), g.prefix + ((size_t)bh * g.nblk + b) * E, C::PRE, pfull(ps_));
            ++npre;
            return true;
        };
        int next = static_cast<int>(atomicAdd(&g.ctl[1], 1u));
        while (ok && next < total) {
            const int u = next;
            next = static_cast<int>(atomicAdd(&g.ctl[1], 1u));
            const int bh = u / g.U2;
            int b, gi;
            unit_block(g, u - bh * g.U2, g.ng_first, g.ng_mid, g.ng_last, b, gi);
            const int fb = block_frame_begin(g, b), fe = block_frame_end(g, b);
            const int L = (fe - fb) * g.HW, nt = (L + kTile - 1) / kTile, ng = ng_of(b);
            const int t_lo = gi * nt / ng, t_hi = (gi + 1) * nt / ng, ntiles = t_hi - t_lo;
            const int nspans = (ntiles + SPAN - 1) / SPAN;
            const int bb = bh / g.H, hh = bh - bb * g.H;
            // the prefix first: it is needed before the group's first tile can be multiplied
            if (!(ok = issue_prefix(bh, b))) break;
            for (int p = 0; p < nspans; ++p, ++kp) {
                const int sl = kp % NLS;
                if (kp >= NLS && !ptx::mbar_wait_bounded(lempty(sl), ((kp / NLS) - 1) & 1, wd, WD_P2_EMPTY, kWaitLimitNs)) {
                    ok = false;
                    break;
                }
                const int t0 = p * SPAN, n = fb * g.HW + (t_lo + t0) * kTile;  // span's first tile and token
                // one record per tile for the epilogue
                for (int h = 0; h < SPAN && t0 + h < ntiles && ok; ++h, ++j) {
                    const int ti = j % C::NINFO;
                    if (j >= C::NINFO &&
                        !ptx::mbar_wait_bounded(tempty(ti), ((j / C::NINFO) - 1) & 1, wd, WD_P2_INFO, kWaitLimitNs)) {
                        ok = false;
                        break;
                    }
                    int *ti_rec = tinfo + 4 * ti;
                    ti_rec[0] = n + h * kTile;
                    ti_rec[1] = bh;
                    ti_rec[2] = min(kTile, L - (t_lo + t0 + h) * kTile);
                    ptx::mbar_arrive(tfull(ti));
                }
                if (!ok) break;
                ScaleSpan sp{};  // NVFP4: the span's scale bytes, rounded outwards to 16 B
                if constexpr (FP4) sp = scale_span<D>((long long)bh * g.N + n, SPAN * kTile, (long long)g.BH * g.N);
                int *inf = linfo + 8 * sl;  // for the transform warps
                inf[0] = u;
                inf[1] = t0;
                inf[2] = ntiles;
                inf[3] = nu;
                inf[4] = n;
                inf[5] = L - (t_lo + t0) * kTile;  // rows of the span inside the block (may exceed the span)
                inf[6] = sp.off;
                const MapCoord mc = map_coord(n, hh, g.swap_q);
                ptx::mbar_arrive_expect_tx(lfull(sl), FP4 ? F::DB + sp.bytes : SPAN * TB);
                ptx::tma_load_4d_hint(ptx::smem_u32(lq(sl)), mq, lfull(sl), 0, mc.y, mc.z, bb, policy);
                if constexpr (FP4) ptx::bulk_load(ptx::smem_u32(lq(sl) + F::DB), g.sq_scale + sp.a0, sp.bytes, lfull(sl));
            }
            ++nu;
        }
        // end markers: transform warps (landing ring) and epilogue (tile ring)
        const int sl = kp % NLS, ti = j % C::NINFO;
        bool marked = false;
        if (ok && (kp < NLS || ptx::mbar_wait_bounded(lempty(sl), ((kp / NLS) - 1) & 1, wd, WD_P2_EMPTY, kWaitLimitNs))) {
            linfo[8 * sl] = kEndFirst;
            ptx::mbar_arrive(lfull(sl));
            marked = true;
        }
        if (ok && (j < C::NINFO ||
                   ptx::mbar_wait_bounded(tempty(ti), ((j / C::NINFO) - 1) & 1, wd, WD_P2_INFO, kWaitLimitNs))) {
            tinfo[4 * ti] = kEndFirst;
            ptx::mbar_arrive(tfull(ti));
        }
        // No bulk write may still be in flight into shared memory when the CTA exits: the
        // last landing of each slot (the end marker's slot was seen released, and its phase
        // moved on) and the last prefix copy.
        const int oldest = marked ? kp - NLS + 1 : kp - NLS;
        for (int kk = kp - 1; kk >= 0 && kk >= oldest; --kk)
            ptx::mbar_wait_bounded(lfull(kk % NLS), (kk / NLS) & 1, wd, WD_P2_FULL, kWaitLimitNs);
        for (int j2 = npre - 1; j2 >= 0 && j2 >= npre - 2; --j2)
            ptx::mbar_wait_bounded(pfull(j2 & 1), (j2 >> 1) & 1, wd, WD_P2_BREADY, kWaitLimitNs);
    }

    // ------------------------------------------------------------ MMA issuer (one thread)
    __device__ void mma() {
        constexpr uint32_t IDESC = ptx::idesc_bf16_f32(128, C::N2, 0, 0);
        for (int k = 0;; ++k) {
            const int so = k % NO, a = k % NA;
            if (ps.flags[0] || !ptx::mbar_wait_bounded(ofull(so), (k / NO) & 1, wd, WD_P2_READY, kWaitLimitNs)) {
                ps.flags[0] = 1;
                break;
            }
            const int *inf = oinfo + 6 * so;
            const int u = ld_volatile(inf), ord = ld_volatile(inf + 3), last = ld_volatile(inf + 5);
            if (u < 0) break;
            if (k >= NA && !ptx::mbar_wait_bounded(acce(a), ((k / NA) - 1) & 1, wd, WD_P2_ACCE, kWaitLimitNs)) {
                ps.flags[0] = 1;
                break;
            }
            ptx::tc_fence_after_sync();
            const uint32_t qa = ptx::smem_u32(oq(so)), pa = ptx::smem_u32(oph(so));
            const uint32_t ba = ptx::smem_u32(bbuf + (ord & 1) * C::IMG);
            const uint32_t dacc = tmem + a * C::ACOLS;
#pragma unroll
            for (int kk = 0; kk < 2 * D / 16; ++kk) {
                // K atom 0 = q~, K atom 1 = phi(q); +32 B per 16-element K step
                const int atom = kk / (D / 16), jj = kk % (D / 16);
                const uint64_t ad = ptx::smem_desc((atom ? pa : qa) + 32 * jj, 16, 8 * ROWB, C::LAYOUT);
                const uint64_t bd = ptx::smem_desc(ba + atom * C::BATOM + 32 * jj, 16, 8 * ROWB, C::LAYOUT);
                ptx::mma_bf16_ss(dacc, ad, bd, IDESC, kk > 0 ? 1u : 0u);
            }
            ptx::mma_commit(tdone(k % NT));
            if (last) ptx::mma_commit(bempty(ord & 1));
        }
        ptx::mma_commit(drain());
        if (!ptx::mbar_wait_bounded(drain(), 0, wd, WD_P2_DRAIN, kWaitLimitNs)) ps.flags[0] = 1;
    }

    // ------------------------------------------------------------ transform warps (one row per thread)
    __device__ void transform(const RopeTab &tab, int r) {
        const int lane = r & 31;
        const int dx = kTile % g.Wg, dy = (kTile / g.Wg) % g.Hg, dt = kTile / g.HW;
        TokPos tp{0, 0, 0};
        int k = 0;  // tiles handed to the MMA so far
        for (int kp = 0;; ++kp) {
            const int sl = kp % NLS;
            if (ps.flags[0] || !ptx::mbar_wait_bounded(lfull(sl), (kp / NLS) & 1, wd, WD_P2_FULL, kWaitLimitNs)) {
                ps.flags[0] = 1;
                break;
            }
            const int *inf = linfo + 8 * sl;
            const int u = ld_volatile(inf), t0 = ld_volatile(inf + 1), ntiles = ld_volatile(inf + 2);
            const int ord = ld_volatile(inf + 3), n = ld_volatile(inf + 4), rows = ld_volatile(inf + 5);
            if (u < 0) {  // pass the end on to the MMA issuer, in operand order
                const int so = k % NO;
                if (k >= NO && !ptx::mbar_wait_bounded(tdone((k - NO) % NT), ((k - NO) / NT) & 1, wd, WD_P2_READY,
                                                       kWaitLimitNs)) {
                    ps.flags[0] = 1;
                    break;
                }
                if (r == 0) oinfo[6 * so] = kEndFirst;
                warp_arrive(ofull(so), lane);
                break;
            }
            const int hmax = min(SPAN, ntiles - t0);
            bool abort = false;
            for (int h = 0; h < hmax; ++h, ++k) {
                const int t = t0 + h, so = k % NO;
                const int valid = min(kTile, rows - h * kTile);
                if (t == 0) {
                    // a new group: build its B operand from the prefix state (the slot's
                    // previous group must be done with it)
                    const int bs = ord & 1;
                    if ((ord >= 2 && !ptx::mbar_wait_bounded(bempty(bs), ((ord >> 1) - 1) & 1, wd, WD_P2_BREADY,
                                                             kWaitLimitNs)) ||
                        !ptx::mbar_wait_bounded(pfull(ord & 1), (ord >> 1) & 1, wd, WD_P2_BREADY, kWaitLimitNs)) {
                        abort = true;
                        break;
                    }
                    const float *pre = reinterpret_cast<const float *>(prefix_buf(ord & 1));
                    uint4 *dst = reinterpret_cast<uint4 *>(bbuf + bs * C::IMG);
                    for (int item = r; item < C::IMG / 16; item += 128) dst[item] = b_operand_chunk<D>(pre, item);
                    // the next bulk copy into the prefix buffer writes through the async proxy
                    ptx::fence_proxy_async_smem();  // also: the B image is read by the MMA (ordered by ofull)
                    warp_arrive(pempty(ord & 1), lane);
                }
                uint32_t w[D / 2], ph[D / 2];
                const bool live = r < valid;
                if constexpr (FP4) {
                    if (live) fp4_row<D>(lq(sl) + r * (D / 2), lq(sl) + F::DB + ld_volatile(inf + 6) + r * F::S1, tabs, w);
                } else {
                    if (live) load_row<D>(lq(sl) + h * TB, r, w);
                }
                if (h == hmax - 1) {
                    // the next TMA into this slot writes through the async proxy: order this
                    // thread's generic reads of the slot before it
                    ptx::fence_proxy_async_smem();
                    warp_arrive(lempty(sl), lane);  // landing slot read
                }
                // operand slot so was last used by tile k - NO: wait for its MMAs
                if (k >= NO && !ptx::mbar_wait_bounded(tdone((k - NO) % NT), ((k - NO) / NT) & 1, wd, WD_P2_READY,
                                                       kWaitLimitNs)) {
                    abort = true;
                    break;
                }
                if (t == 0) tp.init(g, n + h * kTile + r);
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
                    int *oi = oinfo + 6 * so;
                    oi[0] = u;
                    oi[1] = t;
                    oi[3] = ord;
                    oi[5] = t == ntiles - 1;
                }
                warp_arrive(ofull(so), lane);
            }
            if (abort) {
                ps.flags[0] = 1;
                break;
            }
        }
    }

    // ------------------------------------------------------------ epilogue warps (one row per thread)
    // Each warp holds 32 rows of a tile (its TMEM subpartition).  It stages them in shared
    // memory, then writes them out row-major: one store instruction covers 8 rows (d = 32)
    // or 4 (d = 64), 512 bytes that are contiguous when rows are.  No TMA store, so no wait
    // on the copy engine.
    __device__ void epilogue(__nv_bfloat16 *o, int sub, int lane) {
        constexpr int CPR = D / 8;                  // 16-byte chunks per row
        uint8_t *stg = ostg + sub * 32 * ROWB;       // this warp's 32 staged rows (swizzled)
        for (int k = 0;; ++k) {
            const int ti = k % C::NINFO, a = k % NA;
            if (ps.flags[0] || !ptx::mbar_wait_bounded(tfull(ti), (k / C::NINFO) & 1, wd, WD_P2_INFO, kWaitLimitNs)) {
                ps.flags[0] = 1;
                break;
            }
            const int *rec = tinfo + 4 * ti;
            const int n = ld_volatile(rec), bh = ld_volatile(rec + 1), valid = ld_volatile(rec + 2);
            warp_arrive(tempty(ti), lane);
            if (n < 0) break;
            if (!ptx::mbar_wait_bounded(tdone(k % NT), (k / NT) & 1, wd, WD_P2_MMA, kWaitLimitNs)) {
                ps.flags[0] = 1;
                break;
            }
            ptx::tc_fence_after_sync();
            const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * sub) << 16) + a * C::ACOLS;
            // the denominator's two columns and the first 32 numerator columns: one wait
            float v[32], zh, zl;
            ptx::tmem_ld_32_2cols(taddr, taddr + D, v, zh, zl);
            // NVFP4: phi(q) carries the global scale gq (numerator and denominator alike)
            const float gq = FP4 ? g.gq : 1.0f;
            const float inv = FP4 ? __frcp_rn(gq * zh + gq * zl + g.eps) : __frcp_rn(zh + zl + g.eps);
            uint32_t ow[D / 2];
#pragma unroll
            for (int half = 0; half < D / 32; ++half) {
                if (half > 0) ptx::tmem_ld_32cols(taddr + 32 * half, v);
                if constexpr (FP4) {
#pragma unroll
                    for (int q = 0; q < 32; ++q) v[q] *= gq;
                }
#pragma unroll
                for (int q = 0; q < 16; ++q) ow[16 * half + q] = pack_bf16x2(v[2 * q] * inv, v[2 * q + 1] * inv);
            }
            ptx::tc_fence_before_sync();
            warp_arrive(acce(a), lane);  // the accumulator is read: the MMA may overwrite it
            const int bb = bh / g.H, hh = bh - bb * g.H;
            __nv_bfloat16 *obase = o + (size_t)bb * g.lo.batch + (size_t)hh * g.lo.head;
            store_row<D>(stg, lane, ow);
            __syncwarp();
            if (g.lo.tok == D) {  // rows contiguous: the warp's 32 rows are one span
                uint4 *dst = reinterpret_cast<uint4 *>(obase + (size_t)(n + 32 * sub) * D);
#pragma unroll
                for (int i = lane; i < 32 * CPR; i += 32) {
                    const int row = i / CPR, jj = i - row * CPR;
                    if (32 * sub + row < valid)
                        __stcs(dst + i, *reinterpret_cast<const uint4 *>(stg + swz_chunk<D>(row, jj)));
                }
            } else {
#pragma unroll
                for (int i = lane; i < 32 * CPR; i += 32) {
                    const int row = i / CPR, jj = i - row * CPR, nr = 32 * sub + row;
                    if (nr < valid)
                        __stcs(reinterpret_cast<uint4 *>(obase + (size_t)(n + nr) * g.lo.tok) + jj,
                               *reinterpret_cast<const uint4 *>(stg + swz_chunk<D>(row, jj)));
                }
            }
            __syncwarp();  // the staging is read before the next tile's rows go in
        }
    }
};

// ---------------------------------------------------------------------------- kernels
// Shared prologue of both kernels: barriers, TMEM, the RoPE table.  Returns
// this thread's pipeline index `pipe` and its warp index `pw` inside it.
template <typename Cfg>
struct Cta {
    uint8_t *base, *ctrl;
    volatile int *flags;
    float2 *s_tab;
    uint32_t *tmem_slot;
    __device__ explicit Cta(uint8_t *raw, int off_ctrl) {
        base = align1024(raw);
        ctrl = base + off_ctrl;
        flags = reinterpret_cast<volatile int *>(ctrl + Cfg::OFF_FLAGS);
        tmem_slot = reinterpret_cast<uint32_t *>(ctrl + Cfg::OFF_FLAGS + 4);
        s_tab = reinterpret_cast<float2 *>(ctrl + Cfg::CTRL + Cfg::TABS);
    }
    __device__ PipeSmem pipe(int p, int pipe_bytes, uint8_t *ones) const {
        PipeSmem ps;
        ps.base = base + p * pipe_bytes;
        ps.bars = reinterpret_cast<uint64_t *>(ctrl) + p * Cfg::BARS_PER_PIPE;
        ps.info = reinterpret_cast<int *>(ctrl + Cfg::OFF_INFO) + p * Cfg::INFO_PER_PIPE;
        ps.flags = flags;
        ps.ones = ones;
        return ps;
    }
};

// Pass 1: chunk partial states.  Persistent, one CTA per SM, NP pipelines.
template <int D, int PT, int PY, int PX, bool FP4>
__global__ void __launch_bounds__(K1Cfg<D, FP4>::THREADS, 1)
    partial_tc_kernel(const __grid_constant__ CUtensorMap mk, const __grid_constant__ CUtensorMap mv,
                      const __grid_constant__ KGeom g, int *watchdog) {
    using C = K1Cfg<D, FP4>;
    using P = Pass1<D, PT, PY, PX, FP4>;
    extern __shared__ uint8_t smem_raw[];
    Cta<C> cta(smem_raw, C::OFF_CTRL);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int pipe = warp / C::PIPE_WARPS, pw = warp % C::PIPE_WARPS;
    uint8_t *ones = cta.base + C::OFF_ONES;
    if (tid == 0) {
        for (int p = 0; p < C::NP; ++p) P::init_barriers(reinterpret_cast<uint64_t *>(cta.ctrl) + p * C::BARS_PER_PIPE);
        cta.flags[0] = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 0) {
        ptx::tmem_alloc(ptx::smem_u32(cta.tmem_slot), C::TCOLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    const uint32_t tmem_base = *cta.tmem_slot;
    if (tid == 0) griddep_launch_dependents();
    const PipeSmem ps = cta.pipe(pipe, C::PIPE, ones);
    const uint32_t tmem = tmem_base + pipe * C::NA * C::ACOLS;
    uint8_t *tabs = cta.ctrl + C::CTRL;  // NVFP4 decoding tables
    if (pw < 4) {
        const int r = tid & 127, ntrans = 128 * C::NP, tt = pipe * 128 + r;
        const RopeTab tab = load_rope_tab<PT, PY, PX>(g, cta.s_tab, tt, ntrans);
        if constexpr (FP4) fill_fp4_tables(tabs, tt, ntrans);
        uint4 *o4 = reinterpret_cast<uint4 *>(ones);  // all 1.0, so its swizzle is irrelevant
        for (int i = tt; i < C::TB / 16; i += ntrans) o4[i] = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
        ptx::fence_proxy_async_smem();  // the ones block is read by the MMA (async proxy)
        ptx::named_bar_sync(kBarTab, ntrans);
        P(g, ps, watchdog, tmem, tabs).transform(tab, r);
    } else if (pw < 8) {
        P(g, ps, watchdog, tmem, tabs).epilogue(tid & 127, warp & 3);
    } else if (pw == 8) {
        if (lane < 2) P(g, ps, watchdog, tmem, tabs).producer(&mk, &mv, lane);
    } else if (lane == 0) {
        P(g, ps, watchdog, tmem, tabs).mma();
    }
    ptx::tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after_sync();
        ptx::tmem_dealloc(tmem_base, C::TCOLS);
    }
}

// Pass 2: outputs.  Persistent, one CTA per SM, NP pipelines; launched with
// programmatic dependent launch, it reads the prefix states only after
// griddepcontrol.wait (the block scan before it has finished).
template <int D, int PT, int PY, int PX, bool FP4>
__global__ void __launch_bounds__(K2Cfg<D, FP4>::THREADS, 1)
    output_tc_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ KGeom g, __nv_bfloat16 *o,
                     int *watchdog) {
    using C = K2Cfg<D, FP4>;
    using P = Pass2<D, PT, PY, PX, FP4>;
    extern __shared__ uint8_t smem_raw[];
    Cta<C> cta(smem_raw, C::OFF_CTRL);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int pipe = warp / C::PIPE_WARPS, pw = warp % C::PIPE_WARPS;
    if (tid == 0) {
        for (int p = 0; p < C::NP; ++p) P::init_barriers(reinterpret_cast<uint64_t *>(cta.ctrl) + p * C::BARS_PER_PIPE);
        cta.flags[0] = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 0) {
        ptx::tmem_alloc(ptx::smem_u32(cta.tmem_slot), C::TCOLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    const uint32_t tmem_base = *cta.tmem_slot;
    const PipeSmem ps = cta.pipe(pipe, C::PIPE, nullptr);
    const uint32_t tmem = tmem_base + pipe * C::NA * C::ACOLS;
    uint8_t *tabs = cta.ctrl + C::CTRL;  // NVFP4 decoding tables
    if (pw < 4) {
        const int r = tid & 127, ntrans = 128 * C::NP;
        const RopeTab tab = load_rope_tab<PT, PY, PX>(g, cta.s_tab, pipe * 128 + r, ntrans);
        if constexpr (FP4) fill_fp4_tables(tabs, pipe * 128 + r, ntrans);
        ptx::named_bar_sync(kBarTab, ntrans);
        P(g, ps, watchdog, tmem, tabs).transform(tab, r);
    } else if (pw < 8) {
        // pass 1 and the scan, which this kernel may overlap, touch neither Q nor O: only
        // the prefix read (in the producer) waits for them
        P(g, ps, watchdog, tmem, tabs).epilogue(o, warp & 3, lane);
    } else if (pw == 8) {
        if (lane == 0) P(g, ps, watchdog, tmem, tabs).producer(&mq);
    } else if (lane == 0) {
        P(g, ps, watchdog, tmem, tabs).mma();
    }
    ptx::tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after_sync();
        ptx::tmem_dealloc(tmem_base, C::TCOLS);
    }
}

}  // namespace blin
