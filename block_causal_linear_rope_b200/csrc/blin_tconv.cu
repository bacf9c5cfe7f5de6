// Causal block temporal convolution of the Mix-FFN with its one-frame cache.
//
// Talk transcript, causal-FFN passage: in causal training a zero token sits
// between two blocks, so no block sees the next one; a block must see the
// previous one, so that block's last token is cached and placed in front of the
// block.  Per batch entry, pixel and channel, with taps (previous, current, next):
//   y[t] = w0 * x[t-1] + w1 * x[t] + w2 * x[t+1] + bias
// x[t-1] comes from the call or, for the call's first frame, from the cache
// (zero before the video starts); x[t+1] counts only inside the same block of
// F frames and inside the call.  The cache is one frame [B][Hgt*Wid][C]
// whatever the video length.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>

#include "../../include/blin.h"
#include "blin_internal.cuh"

namespace {

constexpr uint64_t kTconvMagic = 0x626c696e54434e56ull;  // "blinTCNV"

// Eight channels of one pixel of one frame: 16 bytes (bf16) or 32 bytes (fp32).
template <typename T>
struct Vec8;
template <>
struct Vec8<__nv_bfloat16> {
    uint4 u;
    __device__ __forceinline__ static Vec8 load(const __nv_bfloat16 *p) {
        Vec8 v;
        v.u = __ldcs(reinterpret_cast<const uint4 *>(p));
        return v;
    }
    __device__ __forceinline__ static Vec8 zero() {
        Vec8 v;
        v.u = make_uint4(0, 0, 0, 0);
        return v;
    }
    __device__ __forceinline__ float get(int i) const {
        const uint32_t w = (&u.x)[i >> 1];
        return __uint_as_float((i & 1) ? (w & 0xFFFF0000u) : (w << 16));
    }
    __device__ __forceinline__ static void store(__nv_bfloat16 *p, const float (&f)[8]) {
        uint4 o;
        uint32_t *w = &o.x;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
            w[i] = *reinterpret_cast<uint32_t *>(&h);
        }
        __stcs(reinterpret_cast<uint4 *>(p), o);
    }
    __device__ __forceinline__ void put(__nv_bfloat16 *p) const { *reinterpret_cast<uint4 *>(p) = u; }
};
template <>
struct Vec8<float> {
    float4 a, b;
    __device__ __forceinline__ static Vec8 load(const float *p) {
        Vec8 v;
        v.a = __ldcs(reinterpret_cast<const float4 *>(p));
        v.b = __ldcs(reinterpret_cast<const float4 *>(p) + 1);
        return v;
    }
    __device__ __forceinline__ static Vec8 zero() {
        Vec8 v;
        v.a = v.b = make_float4(0.f, 0.f, 0.f, 0.f);
        return v;
    }
    __device__ __forceinline__ float get(int i) const { return i < 4 ? (&a.x)[i] : (&b.x)[i - 4]; }
    __device__ __forceinline__ static void store(float *p, const float (&f)[8]) {
        __stcs(reinterpret_cast<float4 *>(p), make_float4(f[0], f[1], f[2], f[3]));
        __stcs(reinterpret_cast<float4 *>(p) + 1, make_float4(f[4], f[5], f[6], f[7]));
    }
    __device__ __forceinline__ void put(float *p) const {
        reinterpret_cast<float4 *>(p)[0] = a;
        reinterpret_cast<float4 *>(p)[1] = b;
    }
};

// One thread per column (batch entry, pixel, 8 channels), walking the call's
// frames with two frames loaded ahead; every element of x is read once and
// every element of y written once.  `cache` (may be NULL) holds frame t0 - 1
// on entry when t0 > 0, and receives the call's last frame when `commit`.
template <typename T>
__global__ void __launch_bounds__(256) tconv_kernel(const T *__restrict__ x, const float *__restrict__ taps,
                                                    const float *__restrict__ bias, T *__restrict__ y, T *cache,
                                                    int B, int Tn, int HW, int C, int t0, int F, int commit) {
    const int C8 = C / 8;
    const long long cols = (long long)B * HW * C8;
    const long long fstride = (long long)HW * C;  // elements between consecutive frames
    for (long long col = blockIdx.x * (long long)blockDim.x + threadIdx.x; col < cols;
         col += (long long)gridDim.x * blockDim.x) {
        const int c8 = (int)(col % C8);
        const long long bs = col / C8;
        const int b = (int)(bs / HW), s = (int)(bs - (long long)b * HW);
        const int c0 = 8 * c8;
        float w0[8], w1[8], w2[8], bb[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            w0[i] = __ldg(taps + 3 * (c0 + i));
            w1[i] = __ldg(taps + 3 * (c0 + i) + 1);
            w2[i] = __ldg(taps + 3 * (c0 + i) + 2);
            bb[i] = bias ? __ldg(bias + c0 + i) : 0.f;
        }
        const T *xc0 = x + ((long long)b * Tn * HW + s) * C + c0;  // frame 0 of this column
        T *yc0 = y + ((long long)b * Tn * HW + s) * C + c0;
        T *cc = cache ? cache + ((long long)b * HW + s) * C + c0 : nullptr;
        Vec8<T> xp = (t0 > 0 && cc) ? Vec8<T>::load(cc) : Vec8<T>::zero();
        Vec8<T> xc = Tn > 0 ? Vec8<T>::load(xc0) : Vec8<T>::zero();
        Vec8<T> x1 = Tn > 1 ? Vec8<T>::load(xc0 + fstride) : Vec8<T>::zero();
        Vec8<T> x2 = Tn > 2 ? Vec8<T>::load(xc0 + 2 * fstride) : Vec8<T>::zero();
        for (int t = 0; t < Tn; ++t) {
            const int ta = t0 + t;
            const bool nxt = t + 1 < Tn && (ta + 1) / F == ta / F;  // the next frame is in this block
            float o[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                float acc = bb[i];
                acc = fmaf(w0[i], xp.get(i), acc);
                acc = fmaf(w1[i], xc.get(i), acc);
                acc = fmaf(w2[i], nxt ? x1.get(i) : 0.f, acc);
                o[i] = acc;
            }
            Vec8<T>::store(yc0 + t * fstride, o);
            xp = xc;
            xc = x1;
            x1 = x2;
            x2 = t + 3 < Tn ? Vec8<T>::load(xc0 + (t + 3) * fstride) : Vec8<T>::zero();
        }
        if (commit && cc && Tn > 0) xp.put(cc);  // the call's last frame (read above) is the new cache
    }
}

blin_status fail(blin_status st, const char *fmt, const char *a = nullptr) {
    char msg[256];
    snprintf(msg, sizeof msg, fmt, a);
    return blin::set_last_error(st, msg);
}

blin_status cuda_fail(cudaError_t e, const char *what) {
    char msg[256];
    snprintf(msg, sizeof msg, "%s: %s", what, cudaGetErrorString(e));
    return blin::set_last_error(BLIN_ERR_CUDA, msg);
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

struct blin_tconv_state {
    uint64_t magic;
    int B, C, HW, device;
    blin_dtype dt;
    void *frame;  // [B][HW][C] in dt: the last frame seen
    int t_next;
    cudaEvent_t last_use;
};

static size_t elem_size(blin_dtype dt) { return dt == BLIN_BF16 ? 2 : 4; }

static blin_status check_tconv_state(const blin_tconv_state *st) {
    if (st == nullptr) return fail(BLIN_ERR_INVALID_ARG, "temporal-conv state is NULL");
    if (st->magic != kTconvMagic) return fail(BLIN_ERR_STATE, "temporal-conv state is not live (freed or foreign)");
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != st->device)
        return fail(BLIN_ERR_STATE, "temporal-conv state lives on another device");
    return BLIN_OK;
}

static blin_status mark_use(blin_tconv_state *st, cudaStream_t s) {
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    cudaError_t e = cudaStreamIsCapturing(s, &cap);
    if (e != cudaSuccess) return cuda_fail(e, "stream capture query");
    if (cap != cudaStreamCaptureStatusNone) return BLIN_OK;
    e = cudaEventRecord(st->last_use, s);
    return e == cudaSuccess ? BLIN_OK : cuda_fail(e, "state event record");
}

extern "C" {

blin_status blin_tconv_state_init(int B, int C, int Hgt, int Wid, blin_dtype dt, blin_stream stream,
                                  blin_tconv_state **out) {
    if (out == nullptr) return fail(BLIN_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    if (B < 1 || C < 1 || Hgt < 1 || Wid < 1) return fail(BLIN_ERR_INVALID_ARG, "B, C, Hgt and Wid must be >= 1");
    if (C % 8) return fail(BLIN_ERR_SHAPE, "C must be a multiple of 8");
    if (dt != BLIN_F32 && dt != BLIN_BF16) return fail(BLIN_ERR_DTYPE, "unknown dtype");
    if ((long long)B * Hgt * Wid * C >= (1LL << 40)) return fail(BLIN_ERR_SHAPE, "cache too large");
    blin_tconv_state *st = new blin_tconv_state{};
    st->magic = kTconvMagic;
    st->B = B;
    st->C = C;
    st->HW = Hgt * Wid;
    st->dt = dt;
    const size_t bytes = (size_t)B * Hgt * Wid * C * elem_size(dt);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaGetDevice(&st->device);
    if (e == cudaSuccess) e = cudaMalloc(&st->frame, bytes);
    if (e == cudaSuccess) e = cudaMemsetAsync(st->frame, 0, bytes, s);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&st->last_use, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventRecord(st->last_use, s);
    if (e != cudaSuccess) {
        if (st->frame) cudaFree(st->frame);
        if (st->last_use) cudaEventDestroy(st->last_use);
        delete st;
        return cuda_fail(e, "temporal-conv state allocation");
    }
    *out = st;
    return BLIN_OK;
}

blin_status blin_tconv_state_free(blin_tconv_state *st) {
    if (st == nullptr) return BLIN_OK;
    if (st->magic != kTconvMagic) return fail(BLIN_ERR_STATE, "temporal-conv state is not live (double free?)");
    int prev = 0;
    cudaGetDevice(&prev);
    cudaSetDevice(st->device);
    const cudaError_t e = cudaEventSynchronize(st->last_use);
    cudaEventDestroy(st->last_use);
    cudaFree(st->frame);
    cudaSetDevice(prev);
    st->magic = 0;
    delete st;
    return e == cudaSuccess ? BLIN_OK : cuda_fail(e, "wait for the state's last use before freeing it");
}

blin_status blin_tconv_state_reset(blin_tconv_state *st, blin_stream stream) {
    blin_status rc = check_tconv_state(st);
    if (rc != BLIN_OK) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const cudaError_t e = cudaMemsetAsync(st->frame, 0, blin_tconv_state_bytes(st), s);
    if (e != cudaSuccess) return cuda_fail(e, "temporal-conv state reset");
    if ((rc = mark_use(st, s)) != BLIN_OK) return rc;
    st->t_next = 0;
    return BLIN_OK;
}

blin_status blin_tconv_state_frame(const blin_tconv_state *st, void **frame, int *t_next) {
    if (st == nullptr) return fail(BLIN_ERR_INVALID_ARG, "temporal-conv state is NULL");
    if (st->magic != kTconvMagic) return fail(BLIN_ERR_STATE, "temporal-conv state is not live");
    if (frame) *frame = st->frame;
    if (t_next) *t_next = st->t_next;
    return BLIN_OK;
}

size_t blin_tconv_state_bytes(const blin_tconv_state *st) {
    if (st == nullptr || st->magic != kTconvMagic) return 0;
    return (size_t)st->B * st->HW * st->C * elem_size(st->dt);
}

blin_status blin_tconv(const void *x, const float *taps, const float *bias, void *y, blin_dtype dt, int B, int C,
                       const blin_geom *g, blin_tconv_state *st, int commit, blin_stream stream) {
    const blin::TraceRange trace("blin_tconv");
    if (g == nullptr) return fail(BLIN_ERR_INVALID_ARG, "geom is NULL");
    if (x == nullptr || y == nullptr || taps == nullptr)
        return fail(BLIN_ERR_INVALID_ARG, "x, taps and y must be non-NULL device pointers");
    if (dt != BLIN_F32 && dt != BLIN_BF16) return fail(BLIN_ERR_DTYPE, "unknown dtype");
    if (B < 1 || C < 1) return fail(BLIN_ERR_INVALID_ARG, "B and C must be >= 1");
    if (C % 8) return fail(BLIN_ERR_SHAPE, "C must be a multiple of 8");
    if (g->T < 0 || g->Hgt < 1 || g->Wid < 1 || g->block_frames < 1)
        return fail(BLIN_ERR_INVALID_ARG, "T must be >= 0; Hgt, Wid and block_frames >= 1");
    if (commit != 0 && commit != 1) return fail(BLIN_ERR_INVALID_ARG, "commit must be 0 or 1");
    if (commit && st == nullptr) return fail(BLIN_ERR_INVALID_ARG, "commit needs a state");
    if (!aligned16(x) || !aligned16(y) || ((reinterpret_cast<uintptr_t>(taps) & 3u) != 0) ||
        (bias != nullptr && (reinterpret_cast<uintptr_t>(bias) & 3u) != 0))
        return fail(BLIN_ERR_ALIGN, "x and y must be 16-byte aligned, taps and bias 4-byte aligned");
    const long long HW = (long long)g->Hgt * g->Wid;
    if (HW >= (1LL << 31) || (long long)B * g->T * HW * C >= (1LL << 40))
        return fail(BLIN_ERR_SHAPE, "problem too large");
    if (st != nullptr) {
        blin_status rc = check_tconv_state(st);
        if (rc != BLIN_OK) return rc;
        if (st->B != B || st->C != C || st->HW != HW || st->dt != dt)
            return fail(BLIN_ERR_STATE, "state shape or dtype differs from the call's");
        if ((long long)st->t_next + g->T >= (1LL << 30)) return fail(BLIN_ERR_SHAPE, "frame index overflow");
    }
    if (g->T == 0) return BLIN_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int t0 = st ? st->t_next : 0;
    const long long cols = (long long)B * HW * (C / 8);
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long blocks = std::min<long long>((cols + 255) / 256, (long long)sms * 8);
    if (dt == BLIN_BF16)
        tconv_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, s>>>(
            static_cast<const __nv_bfloat16 *>(x), taps, bias, static_cast<__nv_bfloat16 *>(y),
            st ? static_cast<__nv_bfloat16 *>(st->frame) : nullptr, B, g->T, (int)HW, C, t0, g->block_frames, commit);
    else
        tconv_kernel<float><<<(unsigned)blocks, 256, 0, s>>>(static_cast<const float *>(x), taps, bias,
                                                              static_cast<float *>(y),
                                                              st ? static_cast<float *>(st->frame) : nullptr, B,
                                                              g->T, (int)HW, C, t0, g->block_frames, commit);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "temporal-conv launch");
    blin::note_launch();
    if (st != nullptr) {
        const blin_status rc = mark_use(st, s);
        if (rc != BLIN_OK) return rc;
        if (commit) st->t_next += g->T;
    }
    return BLIN_OK;
}

}  // extern "C"
