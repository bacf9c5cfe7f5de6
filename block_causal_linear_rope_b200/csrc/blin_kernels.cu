// Device code of libblin's attention path and its launchers.  Besides the
// kernels, this translation unit holds the one device-resident watchdog word
// (g_watchdog); the only other device-resident object of the library is
// blin_prefill_static's scratch array in blin_noalloc.cu.  Host code reaches
// both through cudaGetSymbolAddress, so no relocatable device code is needed.
#include <cuda_bf16.h>

#include <utility>

#include "blin_internal.cuh"

namespace blin {
__device__ int g_watchdog = 0;
}

#include "kern_aux.cuh"
#include "kern_tc.cuh"

namespace blin {

cudaError_t read_and_clear_watchdog(int *code) {
    int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(code, g_watchdog, sizeof(int));
    if (e != cudaSuccess) return e;
    return cudaMemcpyToSymbol(g_watchdog, &zero, sizeof(int));
}

static int *watchdog_ptr() {
    // Address of the current context's watchdog word (a module's device
    // variables exist once per context).
    static ContextCache<int *> cache;
    const unsigned long long ctx = current_context_id();
    int *p = nullptr;
    if (cache.get(ctx, &p)) return p;
    void *a = nullptr;
    if (cudaGetSymbolAddress(&a, g_watchdog) != cudaSuccess) return nullptr;
    cache.put(ctx, static_cast<int *>(a));
    return static_cast<int *>(a);
}

cudaError_t launch_rope_table(const KGeom &g, cudaStream_t s) {
    const int total = g.T * g.pt + g.Hg * g.py + g.Wg * g.px;
    if (total == 0) return cudaSuccess;
    const int threads = 256;
    const int blocks = (total + threads - 1) / threads;
    rope_table_kernel<<<blocks, threads, 0, s>>>(const_cast<float2 *>(g.tab), g.T, g.t0, g.Hg, g.Wg, g.pt, g.py,
                                                 g.px, g.theta);
    return cudaGetLastError();
}

cudaError_t launch_partial_simt(const KGeom &g, int d, bool bf16, const void *k, const void *v,
                                cudaStream_t s) {
    dim3 grid(g.cpb, g.nblk, g.BH);
    if (d == 32) {
        if (bf16)
            partial_simt_kernel<32, __nv_bfloat16><<<grid, 256, 0, s>>>(
                g, static_cast<const __nv_bfloat16 *>(k), static_cast<const __nv_bfloat16 *>(v));
        else
            partial_simt_kernel<32, float><<<grid, 256, 0, s>>>(g, static_cast<const float *>(k),
                                                                static_cast<const float *>(v));
    } else {
        if (bf16)
            partial_simt_kernel<64, __nv_bfloat16><<<grid, 256, 0, s>>>(
                g, static_cast<const __nv_bfloat16 *>(k), static_cast<const __nv_bfloat16 *>(v));
        else
            partial_simt_kernel<64, float><<<grid, 256, 0, s>>>(g, static_cast<const float *>(k),
                                                                static_cast<const float *>(v));
    }
    return cudaGetLastError();
}

cudaError_t launch_output_simt(const KGeom &g, int d, bool bf16, const void *q, void *o,
                               cudaStream_t s) {
    const int max_tok = g.cpb * kChunk;  // >= longest block
    dim3 grid((max_tok + kTile - 1) / kTile, g.nblk, g.BH);
    if (d == 32) {
        if (bf16)
            output_simt_kernel<32, __nv_bfloat16><<<grid, 128, 0, s>>>(
                g, static_cast<const __nv_bfloat16 *>(q), static_cast<__nv_bfloat16 *>(o));
        else
            output_simt_kernel<32, float><<<grid, 128, 0, s>>>(g, static_cast<const float *>(q),
                                                               static_cast<float *>(o));
    } else {
        if (bf16)
            output_simt_kernel<64, __nv_bfloat16><<<grid, 128, 0, s>>>(
                g, static_cast<const __nv_bfloat16 *>(q), static_cast<__nv_bfloat16 *>(o));
        else
            output_simt_kernel<64, float><<<grid, 128, 0, s>>>(g, static_cast<const float *>(q),
                                                               static_cast<float *>(o));
    }
    return cudaGetLastError();
}

// ---------------------------------------------------------------- tensor-core path
// Compiled RoPE splits (pairs per axis): d = 32 -> (8,12,12) dims; d = 64 -> (16,24,24).
bool tc_supported(int d, const int split[3]) {
    if (d == 32) return split[0] == 8 && split[1] == 12 && split[2] == 12;
    if (d == 64) return split[0] == 16 && split[1] == 24 && split[2] == 24;
    return false;
}

// Raise the dynamic shared-memory limit of a kernel (once per context and
// kernel: function attributes belong to a context; the template parameter is
// the kernel itself, not its type).
template <auto Kernel>
static cudaError_t set_smem(int bytes) {
    static ContextCache<int> done;
    const unsigned long long ctx = current_context_id();
    int have = 0;
    if (done.get(ctx, &have) && have >= bytes) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(Kernel, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (e == cudaSuccess) done.put(ctx, 227 * 1024);
    return e;
}

// Largest RoPE table (bytes) the tensor-core kernels can hold in shared memory
// next to their rings (227 KB per CTA).
int tc_table_smem_limit(int d) {
    const int fixed = d == 32 ? std::max(std::max(K1Cfg<32>::FIXED, K2Cfg<32>::FIXED),
                                         std::max(K1Cfg<32, true>::FIXED, K2Cfg<32, true>::FIXED))
                              : std::max(std::max(K1Cfg<64>::FIXED, K2Cfg<64>::FIXED),
                                         std::max(K1Cfg<64, true>::FIXED, K2Cfg<64, true>::FIXED));
    return std::min(24 * 1024, 227 * 1024 - fixed);
}

// Launch with programmatic dependent launch allowed when `pdl`: the kernel may
// start while the previous kernel in the stream finishes; it calls
// griddepcontrol.wait before reading what that kernel wrote.
template <typename... KArgs, typename... Args>
static cudaError_t launch_ex(bool pdl, void (*kernel)(KArgs...), dim3 grid, dim3 block, int smem, cudaStream_t s,
                             Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

cudaError_t launch_scan(const KGeom &g, int d, const float *S_in, const float *z_in, float *S_out,
                        float *z_out, cudaStream_t s) {
    const long long cols = (long long)g.BH * ((d * d + d) / 4);  // (head, float4 column) pairs: one thread each
    const dim3 grid((unsigned)((cols + kScanThreads - 1) / kScanThreads));
    cudaError_t e = launch_ex(true, scan_kernel, grid, dim3(kScanThreads), 0, s, g, d, S_in, z_in, S_out, z_out);
    return e != cudaSuccess ? e : cudaGetLastError();
}

// SMs of the current device (the persistent grid: one CTA per SM).
static int device_sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        n <= 0)
        n = 148;
    return n;
}

// Persistent launch: one CTA per SM, never more CTAs than pipelines have units.
template <auto Kernel, typename... Args>
static cudaError_t launch_persistent(bool pdl, int smem, int threads, long long pipes_needed, int np, cudaStream_t s,
                                     Args &&...args) {
    cudaError_t e = set_smem<Kernel>(smem);
    if (e != cudaSuccess) return e;
    const long long ctas = std::max(1LL, (pipes_needed + np - 1) / np);
    const int grid = (int)std::min<long long>(device_sm_count(), ctas);
    e = launch_ex(pdl, Kernel, dim3(grid), dim3(threads), smem, s, std::forward<Args>(args)...);
    return e != cudaSuccess ? e : cudaGetLastError();
}

template <int D, int PT, int PY, int PX, bool FP4>
static cudaError_t partial_tc(const KGeom &g, const CUtensorMap &mk, const CUtensorMap &mv, int *wd, cudaStream_t s) {
    using C = K1Cfg<D, FP4>;
    const int tab = g.tab_smem ? g.tab_smem_bytes : 0;
    return launch_persistent<partial_tc_kernel<D, PT, PY, PX, FP4>>(false, C::FIXED + tab, C::THREADS,
                                                                     (long long)g.BH * g.U1, C::NP, s, mk, mv, g, wd);
}

template <int D, int PT, int PY, int PX, bool FP4>
static cudaError_t output_tc(const KGeom &g, const CUtensorMap &mq, __nv_bfloat16 *o, int *wd, cudaStream_t s) {
    using C = K2Cfg<D, FP4>;
    const int tab = g.tab_smem ? g.tab_smem_bytes : 0;
    return launch_persistent<output_tc_kernel<D, PT, PY, PX, FP4>>(true, C::FIXED + tab, C::THREADS,
                                                                    (long long)g.BH * g.U2, C::NP, s, mq, g, o, wd);
}

cudaError_t launch_partial_tc(const KGeom &g, int d, bool fp4, const CUtensorMap &mk, const CUtensorMap &mv,
                              cudaStream_t s) {
    int *wd = watchdog_ptr();
    if (wd == nullptr) return cudaErrorInvalidDevice;
    if (d == 32)
        return fp4 ? partial_tc<32, 4, 6, 6, true>(g, mk, mv, wd, s) : partial_tc<32, 4, 6, 6, false>(g, mk, mv, wd, s);
    return fp4 ? partial_tc<64, 8, 12, 12, true>(g, mk, mv, wd, s) : partial_tc<64, 8, 12, 12, false>(g, mk, mv, wd, s);
}

cudaError_t launch_output_tc(const KGeom &g, int d, bool fp4, const CUtensorMap &mq, void *o, cudaStream_t s) {
    int *wd = watchdog_ptr();
    if (wd == nullptr) return cudaErrorInvalidDevice;
    __nv_bfloat16 *ob = static_cast<__nv_bfloat16 *>(o);
    if (d == 32)
        return fp4 ? output_tc<32, 4, 6, 6, true>(g, mq, ob, wd, s) : output_tc<32, 4, 6, 6, false>(g, mq, ob, wd, s);
    return fp4 ? output_tc<64, 8, 12, 12, true>(g, mq, ob, wd, s) : output_tc<64, 8, 12, 12, false>(g, mq, ob, wd, s);
}

}  // namespace blin
