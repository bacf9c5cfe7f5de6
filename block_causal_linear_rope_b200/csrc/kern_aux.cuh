// RoPE cos/sin table, fixed-order chunk reduction + inclusive block scan, and
// the fp32 CUDA-core path (any RoPE split, fp32 or bf16 storage).
#pragma once

#include <cuda_bf16.h>

#include "blin_internal.cuh"

namespace blin {

// ---------------------------------------------------------------- RoPE table
// Entry i of the (cos, sin) table of a call: [T][pt] (absolute frames
// t0..t0+T-1), then [Hg][py], then [Wg][px]; pair j of an axis with d_a dims
// turns by p * theta^(-2j/d_a).  Angle and sin/cos are taken in double, then
// rounded to float.  (3D RoPE for linear attention: SANA-Video talk transcript.)
__device__ __forceinline__ float2 rope_entry(int i, int T, int t0, int Hg, int pt, int py, int px, double theta) {
    const int nt = T * pt, ny = Hg * py;
    int pos, j, pairs;
    if (i < nt) {
        pos = t0 + i / pt;
        j = i % pt;
        pairs = pt;
    } else if (i < nt + ny) {
        const int r = i - nt;
        pos = r / py;
        j = r % py;
        pairs = py;
    } else {
        const int r = i - nt - ny;
        pos = r / px;
        j = r % px;
        pairs = px;
    }
    const double freq = pow(theta, -2.0 * static_cast<double>(j) / static_cast<double>(2 * pairs));
    double s, c;
    sincos(static_cast<double>(pos) * freq, &s, &c);
    return make_float2(static_cast<float>(c), static_cast<float>(s));
}

// Whole table in global memory (CUDA-core path).
__global__ void rope_table_kernel(float2 *tab, int T, int t0, int Hg, int Wg, int pt, int py, int px,
                                  double theta) {
    const int total = T * pt + Hg * py + Wg * px;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += gridDim.x * blockDim.x)
        tab[i] = rope_entry(i, T, t0, Hg, pt, py, px, theta);
}

// ---------------------------------------------------------------- block scan
// For each head and each element e of (S | z):
//   P_b    = ((part_b0 + part_b1) + part_b2) + ...        (chunks of block b, fixed order)
//   S_<=b  = S_<=b-1 + P_b,  S_<=-1 = S_in (or 0)
// written to prefix[bh][b][e]; the last one also to S_out (may alias S_in).
// The order depends only on the block's own length, so a block-by-block
// stream reproduces a one-shot prefill bit for bit.  (Talk transcript: the
// new state is the cached state plus the block's contribution.)
// One thread per (head, float4 column), all heads' columns laid end to end, in
// 128-thread CTAs so that every SM takes a share.
constexpr int kScanLoads = 8;  // chunk partial loads in flight per thread (a block's chunks, in groups)
constexpr int kScanThreads = 128;

__device__ __forceinline__ float4 f4add(float4 a, float4 b) {
    return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}

// Each thread walks its column block by block: a block's chunk partials are loaded
// together (up to kScanLoads at a time) and summed in chunk order, then added to the
// running state.
__global__ void __launch_bounds__(kScanThreads) scan_kernel(KGeom g, int d, const float *S_in, const float *z_in,
                                                             float *S_out, float *z_out) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");  // chunk partials come from the previous kernel
    const int E4 = (d * d + d) / 4;
    const long long f = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (f >= (long long)g.BH * E4) return;
    const int bh = (int)(f / E4), e4 = (int)(f - (long long)bh * E4);
    const float4 *part = reinterpret_cast<const float4 *>(g.part) + (size_t)bh * g.nblk * g.cpb * E4 + e4;
    float4 *prefix = reinterpret_cast<float4 *>(g.prefix) + (size_t)bh * g.nblk * E4 + e4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (S_in != nullptr)
        acc = 4 * e4 < d * d ? reinterpret_cast<const float4 *>(S_in + (size_t)bh * d * d)[e4]
                             : reinterpret_cast<const float4 *>(z_in + (size_t)bh * d)[e4 - d * d / 4];
    for (int b = 0; b < g.nblk; ++b) {
        const int nc = units_of_block(g, b, g.nc_first, g.nc_mid, g.nc_last);
        const float4 *src = part + (size_t)b * g.cpb * E4;
        float4 pb = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int c0 = 0; c0 < nc; c0 += kScanLoads) {
            float4 v[kScanLoads];
#pragma unroll
            for (int j = 0; j < kScanLoads; ++j)
                if (c0 + j < nc) v[j] = __ldcg(src + (size_t)(c0 + j) * E4);
#pragma unroll
            for (int j = 0; j < kScanLoads; ++j)
                if (c0 + j < nc) pb = c0 + j == 0 ? v[j] : f4add(pb, v[j]);
        }
        acc = f4add(acc, pb);  // block b complete
        prefix[(size_t)b * E4] = acc;
    }
    if (S_out != nullptr) {
        if (4 * e4 < d * d)
            reinterpret_cast<float4 *>(S_out + (size_t)bh * d * d)[e4] = acc;
        else
            reinterpret_cast<float4 *>(z_out + (size_t)bh * d)[e4 - d * d / 4] = acc;
    }
}

// ---------------------------------------------------------------- helpers
__device__ __forceinline__ float load_val(const float *p, size_t i) { return p[i]; }
__device__ __forceinline__ float load_val(const __nv_bfloat16 *p, size_t i) {
    return __bfloat162float(p[i]);
}
__device__ __forceinline__ void store_val(float *p, size_t i, float x) { p[i] = x; }
__device__ __forceinline__ void store_val(__nv_bfloat16 *p, size_t i, float x) {
    p[i] = __float2bfloat16_rn(x);
}

// Element offset of token `tok` of head `bh` (= b * H + h) in a strided operand.
__device__ __forceinline__ size_t row_off(const Layout &l, int H, int bh, int tok) {
    const int b = bh / H, h = bh - b * H;
    return (size_t)b * l.batch + (size_t)h * l.head + (size_t)tok * l.tok;
}

// (cos, sin) of RoPE pair p (0 <= p < d/2) at relative frame t, row y, column x.
__device__ __forceinline__ float2 rope_cs(const KGeom &g, int p, int t, int y, int x) {
    if (p < g.pt) return g.tab[t * g.pt + p];
    p -= g.pt;
    if (p < g.py) return g.tab[g.tab_y + y * g.py + p];
    p -= g.py;
    return g.tab[g.tab_x + x * g.px + p];
}

// ---------------------------------------------------------------- SIMT partial states
// One CTA per (chunk, block, head): P = sum_m (R_m phi(k_m)) v_m^T and
// zp = sum_m phi(k_m) over the chunk's tokens, in fp32 FMAs.
template <int D, typename Tin>
__global__ void __launch_bounds__(256) partial_simt_kernel(KGeom g, const Tin *k, const Tin *v) {
    constexpr int SUB = 32;
    constexpr int PER = D * D / 256;
    __shared__ float kr[SUB][D + 1], kp[SUB][D + 1], vv[SUB][D + 1];
    const int c = blockIdx.x, b = blockIdx.y, bh = blockIdx.z;
    const int fb = block_frame_begin(g, b), fe = block_frame_end(g, b);
    const int tok0 = fb * g.HW, ntok = (fe - fb) * g.HW;
    const int cs = c * kChunk;
    if (cs >= ntok) return;
    const int ce = min(ntok, cs + kChunk);
    float acc[PER];
#pragma unroll
    for (int q = 0; q < PER; ++q) acc[q] = 0.0f;
    float zacc = 0.0f;
    for (int t = cs; t < ce; t += SUB) {
        const int n = min(SUB, ce - t);
        for (int idx = threadIdx.x; idx < SUB * (D / 2); idx += blockDim.x) {
            const int r = idx / (D / 2), p = idx % (D / 2);
            float a = 0.f, bb = 0.f, ra = 0.f, rb = 0.f, va = 0.f, vb = 0.f;
            if (r < n) {
                const int tok = tok0 + t + r;
                const size_t off = row_off(g.lq, g.H, bh, tok) + 2 * p;
                a = fmaxf(load_val(k, off), 0.f);
                bb = fmaxf(load_val(k, off + 1), 0.f);
                va = load_val(v, off);
                vb = load_val(v, off + 1);
                const int tt = tok / g.HW, rem = tok - tt * g.HW, y = rem / g.Wg, x = rem - y * g.Wg;
                const float2 cs2 = rope_cs(g, p, tt, y, x);
                ra = a * cs2.x - bb * cs2.y;
                rb = a * cs2.y + bb * cs2.x;
            }
            kr[r][2 * p] = ra;
            kr[r][2 * p + 1] = rb;
            kp[r][2 * p] = a;
            kp[r][2 * p + 1] = bb;
            vv[r][2 * p] = va;
            vv[r][2 * p + 1] = vb;
        }
        __syncthreads();
#pragma unroll
        for (int q = 0; q < PER; ++q) {
            const int e = threadIdx.x + q * 256, i = e / D, j = e % D;
            float s = acc[q];
            for (int r = 0; r < n; ++r) s = fmaf(kr[r][i], vv[r][j], s);
            acc[q] = s;
        }
        if (threadIdx.x < D)
            for (int r = 0; r < n; ++r) zacc += kp[r][threadIdx.x];
        __syncthreads();
    }
    float *out = g.part + ((size_t)(bh * g.nblk + b) * g.cpb + c) * (D * D + D);
#pragma unroll
    for (int q = 0; q < PER; ++q) out[threadIdx.x + q * 256] = acc[q];
    if (threadIdx.x < D) out[D * D + threadIdx.x] = zacc;
}

// ---------------------------------------------------------------- SIMT output
// One thread per query token: o = (R phi(q))^T S_<=b / (phi(q) . z_<=b + eps).
template <int D, typename Tin>
__global__ void __launch_bounds__(128) output_simt_kernel(KGeom g, const Tin *q, Tin *o) {
    __shared__ float S[D][D];
    __shared__ float z[D];
    const int tile = blockIdx.x, b = blockIdx.y, bh = blockIdx.z;
    const int fb = block_frame_begin(g, b), fe = block_frame_end(g, b);
    const int tok0 = fb * g.HW, ntok = (fe - fb) * g.HW;
    const int ts = tile * kTile;
    if (ts >= ntok) return;
    const float *pre = g.prefix + ((size_t)bh * g.nblk + b) * (D * D + D);
    for (int e = threadIdx.x; e < D * D; e += blockDim.x) S[e / D][e % D] = pre[e];
    if (threadIdx.x < D) z[threadIdx.x] = pre[D * D + threadIdx.x];
    __syncthreads();
    const int r = ts + threadIdx.x;
    if (r >= ntok) return;
    const int tok = tok0 + r;
    const size_t off = row_off(g.lq, g.H, bh, tok), ooff = row_off(g.lo, g.H, bh, tok);
    const int tt = tok / g.HW, rem = tok - tt * g.HW, y = rem / g.Wg, x = rem - y * g.Wg;
    float rq[D];
    float den = 0.f;
#pragma unroll
    for (int p = 0; p < D / 2; ++p) {
        const float a = fmaxf(load_val(q, off + 2 * p), 0.f);
        const float bb = fmaxf(load_val(q, off + 2 * p + 1), 0.f);
        den = fmaf(a, z[2 * p], den);
        den = fmaf(bb, z[2 * p + 1], den);
        const float2 cs2 = rope_cs(g, p, tt, y, x);
        rq[2 * p] = a * cs2.x - bb * cs2.y;
        rq[2 * p + 1] = a * cs2.y + bb * cs2.x;
    }
    den += g.eps;
#pragma unroll 4
    for (int j = 0; j < D; ++j) {
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < D; ++i) s = fmaf(rq[i], S[i][j], s);
        store_val(o, ooff + j, s / den);
    }
}

}  // namespace blin
