// Tensor-core path for bf16 Q/K/V on sm_100a (d = 32 or 64).
//
// Pass 1 (partial_tc_kernel): per (chunk of <= 1024 tokens, block, head) a CTA
//   streams 128-token K and V tiles into shared memory with TMA (64B/128B
//   swizzle), overwrites each K row in place with R_m phi(k_m) (bf16),
//   accumulates phi(k_m) in fp32 registers, and lets tcgen05.mma accumulate
//   P = K~^T V in TMEM (M = 64 rows of K~^T, N = d columns of V, K = tokens).
//   Both operands are MN-major views of the token-major tiles, so no
//   transpose is ever materialised.
// Pass 2 (output_tc_kernel): per (up to 8 tiles of 128 queries, block, head)
//   the CTA converts S_<=b to a bf16 K-major B operand once, streams Q tiles
//   with TMA, overwrites each row with R_n phi(q_n) (bf16) while taking
//   den = phi(q_n) . z_<=b + eps in fp32, runs num = Q~ S_<=b on tcgen05
//   (M = 128 tokens, N = d, K = d), reads num back from TMEM, divides, and
//   stores bf16 rows with a TMA store (or plain stores for a ragged tile).
//
// Warp roles: warps 0-3 own one token row each per tile (thread r <-> row r;
// they also read TMEM lanes 32w..32w+31); warp 4 lane 0 issues the TMA loads.
// Thread 0 issues MMAs.  All waits are bounded (see ptx::mbar_wait_bounded).
#pragma once

#include <cuda_bf16.h>

#include "blin_internal.cuh"
#include "ptx_sm100.cuh"

namespace blin {

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s: far beyond any legitimate wait

template <int D>
struct TcCfg {
    static constexpr int ROWB = D * 2;                  // bytes per token row (bf16)
    static constexpr int TB = kTile * ROWB;             // bytes per 128-row tile
    static constexpr uint32_t LAYOUT = D == 32 ? 4u : 2u;  // 64B : 128B swizzle
    static constexpr int P1_STAGES = D == 32 ? 4 : 3;
    static constexpr int P2_STAGES = 4;
};

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

// phi (ReLU) then 3D RoPE of one token row held as D/2 bf16x2 words (pair p =
// features 2p, 2p+1, low half = even feature).  Optionally accumulates the
// unrotated phi into zp and the unrotated phi . z into den.
// (RoPE inside linear attention: talk transcript; RoPE only in the numerator,
// phi . z without RoPE in the denominator: news article, positional encoding.)
template <int D, int PT, int PY, int PX, bool ZP, bool DEN>
__device__ __forceinline__ void phi_rope_row(uint32_t (&w)[D / 2], const KGeom &g, const TokPos &tp,
                                             float (&zp)[D], float &den, const float *zs) {
    static_assert(PT + PY + PX == D / 2, "split must cover d");
    const float2 *rt = g.tab + tp.t * PT;
    const float2 *ry = g.tab + g.tab_y + tp.y * PY;
    const float2 *rx = g.tab + g.tab_x + tp.x * PX;
#pragma unroll
    for (int p = 0; p < D / 2; ++p) {
        const float2 cs = p < PT ? __ldg(rt + p) : (p < PT + PY ? __ldg(ry + (p - PT)) : __ldg(rx + (p - PT - PY)));
        const float a = fmaxf(__uint_as_float(w[p] << 16), 0.f);
        const float b = fmaxf(__uint_as_float(w[p] & 0xFFFF0000u), 0.f);
        if constexpr (ZP) {
            zp[2 * p] += a;
            zp[2 * p + 1] += b;
        }
        if constexpr (DEN) {
            den = fmaf(a, zs[2 * p], den);
            den = fmaf(b, zs[2 * p + 1], den);
        }
        const float ra = fmaf(a, cs.x, -b * cs.y);
        const float rb = fmaf(a, cs.y, b * cs.x);
        w[p] = pack_bf16x2(ra, rb);
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

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

template <int D>
constexpr int partial_tc_smem_bytes() {
    return TcCfg<D>::P1_STAGES * 2 * TcCfg<D>::TB + 1024 + 256;
}
template <int D>
constexpr int output_tc_smem_bytes() {
    return TcCfg<D>::P2_STAGES * TcCfg<D>::TB + D * TcCfg<D>::ROWB + D * 4 + 1024 + 256;
}

// =========================================================================== pass 1
template <int D, int PT, int PY, int PX>
__global__ void __launch_bounds__(160, 1)
    partial_tc_kernel(const __grid_constant__ CUtensorMap mk, const __grid_constant__ CUtensorMap mv,
                      KGeom g, int *watchdog) {
    using C = TcCfg<D>;
    constexpr int NS = C::P1_STAGES;
    constexpr int TB = C::TB, ROWB = C::ROWB;
    constexpr uint32_t IDESC = ptx::idesc_bf16_f32(64, D, 1, 1);
    constexpr uint32_t TCOLS = D;  // 64 x D fp32 accumulator (M = 64 layout: lanes 0-15 of each subpartition)

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + NS * 2 * TB);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * NS + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    auto ktile = [&](int s) { return smem + s * 2 * TB; };
    auto vtile = [&](int s) { return smem + s * 2 * TB + TB; };
    auto full = [&](int s) { return ptx::smem_u32(bars + s); };
    auto empty = [&](int s) { return ptx::smem_u32(bars + NS + s); };
    const uint32_t accbar = ptx::smem_u32(bars + 2 * NS);

    const int c = blockIdx.x, b = blockIdx.y, bh = blockIdx.z;
    const int fb = block_frame_begin(g, b), fe = block_frame_end(g, b);
    const int btok0 = fb * g.HW, bntok = (fe - fb) * g.HW;
    const int cs = c * kChunk;
    if (cs >= bntok) return;  // CTA-uniform, before any barrier or TMEM use
    const int clen = min(kChunk, bntok - cs);
    const int ntiles = (clen + kTile - 1) / kTile;
    const int row0 = bh * g.N + btok0 + cs;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            ptx::mbar_init(full(s), 1);
            ptx::mbar_init(empty(s), 1);
        }
        ptx::mbar_init(accbar, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 0) {
        ptx::tmem_alloc(ptx::smem_u32(tmem_slot), TCOLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == 4) {
        if (lane == 0) {
            ptx::tma_prefetch_map(&mk);
            ptx::tma_prefetch_map(&mv);
            for (int i = 0; i < ntiles; ++i) {
                const int s = i % NS;
                // on timeout just stop issuing: the compute warps then time out on
                // `full` themselves and agree on the abort across their barrier
                if (i >= NS &&
                    !ptx::mbar_wait_bounded(empty(s), ((i / NS) - 1) & 1, watchdog, WD_PARTIAL_EMPTY,
                                            kWaitLimitNs))
                    break;
                ptx::mbar_arrive_expect_tx(full(s), 2 * TB);
                ptx::tma_load_2d(ptx::smem_u32(ktile(s)), &mk, full(s), 0, row0 + i * kTile);
                ptx::tma_load_2d(ptx::smem_u32(vtile(s)), &mv, full(s), 0, row0 + i * kTile);
            }
        }
    } else {
        const int r = tid;  // token row owned by this thread
        TokPos tp;
        tp.init(g, btok0 + cs + r);
        const int dx = kTile % g.Wg, dy = (kTile / g.Wg) % g.Hg, dt = kTile / g.HW;
        float zp[D];
#pragma unroll
        for (int i = 0; i < D; ++i) zp[i] = 0.f;
        float unused_den = 0.f;
        bool ok = true;
        for (int i = 0; i < ntiles; ++i) {
            const int s = i % NS;
            ok = ptx::mbar_wait_bounded(full(s), (i / NS) & 1, watchdog, WD_PARTIAL_FULL, kWaitLimitNs);
            if (!ok) *abort_flag = 1;
            if (ok) {
                if (i * kTile + r < clen) {
                    uint32_t w[D / 2];
                    load_row<D>(ktile(s), r, w);
                    phi_rope_row<D, PT, PY, PX, true, false>(w, g, tp, zp, unused_den, nullptr);
                    store_row<D>(ktile(s), r, w);
                } else {
                    // rows past the chunk: zero both operands so they add nothing
                    zero_row<D>(ktile(s), r);
                    zero_row<D>(vtile(s), r);
                }
            }
            ptx::fence_proxy_async_smem();
            ptx::named_bar_sync(1, 128);
            if (*abort_flag) { ok = false; break; }
            if (r == 0) {
                ptx::tc_fence_after_sync();
                const uint32_t ka = ptx::smem_u32(ktile(s)), va = ptx::smem_u32(vtile(s));
#pragma unroll
                for (int kk = 0; kk < kTile / 16; ++kk) {
                    // A = K~^T: MN-major, 8-token groups every 8 rows; for d = 32 the
                    // second 32-row M atom (rows 32..63, unused) is the V tile at +TB.
                    const uint64_t ad = ptx::smem_desc(ka + kk * 16 * ROWB, TB, 8 * ROWB, C::LAYOUT);
                    const uint64_t bd = ptx::smem_desc(va + kk * 16 * ROWB, TB, 8 * ROWB, C::LAYOUT);
                    ptx::mma_bf16_ss(tmem, ad, bd, IDESC, (i > 0 || kk > 0) ? 1u : 0u);
                }
                ptx::mma_commit(empty(s));
                if (i == ntiles - 1) ptx::mma_commit(accbar);
            }
            tp.advance(g, dx, dy, dt);
        }
        // ---- epilogue: P from TMEM, zp via a fixed-order shared-memory reduction
        float *out = g.part + ((size_t)(bh * g.nblk + b) * g.cpb + c) * (D * D + D);
        if (ok) ok = ptx::mbar_wait_bounded(accbar, 0, watchdog, WD_PARTIAL_ACC, kWaitLimitNs);
        ptx::tc_fence_after_sync();
        {
            // M = 64 accumulator: row m lives in TMEM lane (m % 16) + 32 * (m / 16).
            // tcgen05.ld is warp-collective, so only the store depends on `ok`.
            const int m = 16 * warp + lane;
            if (D == 64 || warp < 2) {
#pragma unroll
                for (int half = 0; half < D / 32; ++half) {
                    float v[32];
                    ptx::tmem_ld_32cols(tmem + (static_cast<uint32_t>(32 * warp) << 16) + 32 * half, v);
                    if (ok && lane < 16) {
                        float4 *dst = reinterpret_cast<float4 *>(out + m * D + 32 * half);
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
                    }
                }
            }
        }
        ptx::tc_fence_before_sync();
        ptx::named_bar_sync(1, 128);
        // stage memory is idle now (all loads consumed, all MMAs complete)
        float *red = reinterpret_cast<float *>(smem);
#pragma unroll
        for (int i = 0; i < D; ++i) red[r * (D + 1) + i] = zp[i];
        ptx::named_bar_sync(1, 128);
        if (ok && r < D) {
            float s = 0.f;
            for (int t = 0; t < kTile; ++t) s += red[t * (D + 1) + r];
            out[D * D + r] = s;
        }
    }
    ptx::tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after_sync();
        ptx::tmem_dealloc(tmem, TCOLS);
    }
}

// =========================================================================== pass 2
template <int D, int PT, int PY, int PX>
__global__ void __launch_bounds__(160, 1)
    output_tc_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mo,
                     KGeom g, __nv_bfloat16 *o, int *watchdog) {
    using C = TcCfg<D>;
    constexpr int NS = C::P2_STAGES;
    constexpr int TB = C::TB, ROWB = C::ROWB;
    constexpr uint32_t IDESC = ptx::idesc_bf16_f32(128, D, 0, 0);
    constexpr uint32_t TCOLS = 2 * D;  // two 128 x D fp32 accumulators

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *sop = smem + NS * TB;  // S_<=b as bf16, K-major B operand: row n = value feature j
    float *zs = reinterpret_cast<float *>(sop + D * ROWB);
    uint64_t *bars = reinterpret_cast<uint64_t *>(zs + D);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * NS + 2);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    auto qtile = [&](int s) { return smem + s * TB; };
    auto full = [&](int s) { return ptx::smem_u32(bars + s); };
    auto empty = [&](int s) { return ptx::smem_u32(bars + NS + s); };
    auto mmad = [&](int a) { return ptx::smem_u32(bars + 2 * NS + a); };

    const int c = blockIdx.x, b = blockIdx.y, bh = blockIdx.z;
    const int fb = block_frame_begin(g, b), fe = block_frame_end(g, b);
    const int btok0 = fb * g.HW, bntok = (fe - fb) * g.HW;
    const int qs = c * kQTiles * kTile;
    if (qs >= bntok) return;  // CTA-uniform
    const int qlen = min(kQTiles * kTile, bntok - qs);
    const int ntiles = (qlen + kTile - 1) / kTile;
    const int row0 = bh * g.N + btok0 + qs;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            ptx::mbar_init(full(s), 1);
            ptx::mbar_init(empty(s), 1);
        }
        ptx::mbar_init(mmad(0), 1);
        ptx::mbar_init(mmad(1), 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 0) {
        ptx::tmem_alloc(ptx::smem_u32(tmem_slot), TCOLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == 4) {
        if (lane == 0) {
            ptx::tma_prefetch_map(&mq);
            ptx::tma_prefetch_map(&mo);
            for (int i = 0; i < ntiles; ++i) {
                const int s = i % NS;
                if (i >= NS &&
                    !ptx::mbar_wait_bounded(empty(s), ((i / NS) - 1) & 1, watchdog, WD_OUT_EMPTY,
                                            kWaitLimitNs))
                    break;
                ptx::mbar_arrive_expect_tx(full(s), TB);
                ptx::tma_load_2d(ptx::smem_u32(qtile(s)), &mq, full(s), 0, row0 + i * kTile);
            }
        }
    } else {
        const int r = tid;
        // ---- prologue: S_<=b (fp32, row i = key feature) -> bf16 B operand with
        // row n = value feature j holding S[0..D)[j] (K-major, swizzled); z to smem.
        const float *pre = g.prefix + ((size_t)bh * g.nblk + b) * (D * D + D);
        for (int item = r; item < D * (D / 8); item += 128) {
            const int j = item / (D / 8), gq = item % (D / 8);
            uint32_t w4[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                w4[u] = pack_bf16x2(pre[(8 * gq + 2 * u) * D + j], pre[(8 * gq + 2 * u + 1) * D + j]);
            *reinterpret_cast<uint4 *>(sop + swz_chunk<D>(j, gq)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
        if (r < D) zs[r] = pre[D * D + r];
        ptx::fence_proxy_async_smem();
        ptx::named_bar_sync(1, 128);

        TokPos tp;
        tp.init(g, btok0 + qs + r);
        const int dx = kTile % g.Wg, dy = (kTile / g.Wg) % g.Hg, dt = kTile / g.HW;
        float zp_unused[D];
        const uint32_t sop_a = ptx::smem_u32(sop);
        for (int i = 0; i < ntiles; ++i) {
            const int s = i % NS, acc = i & 1;
            bool ok = ptx::mbar_wait_bounded(full(s), (i / NS) & 1, watchdog, WD_OUT_FULL, kWaitLimitNs);
            if (!ok) *abort_flag = 1;
            const bool valid = ok && (i * kTile + r < qlen);
            float den = 0.f;
            if (valid) {
                uint32_t w[D / 2];
                load_row<D>(qtile(s), r, w);
                phi_rope_row<D, PT, PY, PX, false, true>(w, g, tp, zp_unused, den, zs);
                store_row<D>(qtile(s), r, w);
            }
            den += g.eps;
            ptx::fence_proxy_async_smem();
            ptx::named_bar_sync(1, 128);
            if (*abort_flag) break;
            if (r == 0) {
                ptx::tc_fence_after_sync();
                const uint32_t qa = ptx::smem_u32(qtile(s));
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    // K-major: +32 B per 16-element K step inside the swizzled row
                    const uint64_t ad = ptx::smem_desc(qa + kk * 32, 16, 8 * ROWB, C::LAYOUT);
                    const uint64_t bd = ptx::smem_desc(sop_a + kk * 32, 16, 8 * ROWB, C::LAYOUT);
                    ptx::mma_bf16_ss(tmem + acc * D, ad, bd, IDESC, kk > 0 ? 1u : 0u);
                }
                ptx::mma_commit(mmad(acc));
            }
            ok = ptx::mbar_wait_bounded(mmad(acc), (i >> 1) & 1, watchdog, WD_OUT_MMA, kWaitLimitNs);
            if (!ok) *abort_flag = 1;
            ptx::tc_fence_after_sync();
            const bool full_tile = (i + 1) * kTile <= qlen;
            const float inv = __frcp_rn(den);
            {  // tcgen05.ld is warp-collective: executed by every lane, stores gated by `valid`
#pragma unroll
                for (int half = 0; half < D / 32; ++half) {
                    float v[32];
                    ptx::tmem_ld_32cols(tmem + (static_cast<uint32_t>(32 * warp) << 16) + acc * D + 32 * half, v);
                    uint32_t ow[16];
#pragma unroll
                    for (int u = 0; u < 16; ++u) ow[u] = pack_bf16x2(v[2 * u] * inv, v[2 * u + 1] * inv);
                    if (valid && ok) {
                        if (full_tile) {
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                *reinterpret_cast<uint4 *>(qtile(s) + swz_chunk<D>(r, 4 * half + j)) =
                                    make_uint4(ow[4 * j], ow[4 * j + 1], ow[4 * j + 2], ow[4 * j + 3]);
                        } else {
                            uint4 *dst = reinterpret_cast<uint4 *>(o + ((size_t)row0 + i * kTile + r) * D + 32 * half);
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                dst[j] = make_uint4(ow[4 * j], ow[4 * j + 1], ow[4 * j + 2], ow[4 * j + 3]);
                        }
                    }
                }
            }
            ptx::tc_fence_before_sync();
            ptx::fence_proxy_async_smem();
            ptx::named_bar_sync(1, 128);
            if (*abort_flag) break;
            if (r == 0) {
                if (full_tile) {
                    ptx::tma_store_2d(&mo, ptx::smem_u32(qtile(s)), 0, row0 + i * kTile);
                    ptx::bulk_commit_group();
                    ptx::bulk_wait_group_read<0>();
                }
                ptx::mbar_arrive(empty(s));
            }
            tp.advance(g, dx, dy, dt);
        }
        if (r == 0) ptx::bulk_wait_group<0>();
    }
    ptx::tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after_sync();
        ptx::tmem_dealloc(tmem, TCOLS);
    }
}

}  // namespace blin
