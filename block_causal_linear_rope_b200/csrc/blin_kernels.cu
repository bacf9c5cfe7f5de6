// All device code of libblin lives in this translation unit (one watchdog word
// per device, no relocatable device code needed) together with its launchers.
#include <cuda_bf16.h>

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
    // Address of this device's watchdog word (cached per device).
    static int *ptrs[64] = {nullptr};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    if (ptrs[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_watchdog) != cudaSuccess) return nullptr;
        ptrs[dev] = static_cast<int *>(p);
    }
    return ptrs[dev];
}

cudaError_t launch_rope_table(const KGeom &g, double theta, cudaStream_t s) {
    const int total = g.T * g.pt + g.Hg * g.py + g.Wg * g.px;
    if (total == 0) return cudaSuccess;
    const int threads = 256;
    const int blocks = (total + threads - 1) / threads;
    rope_table_kernel<<<blocks, threads, 0, s>>>(const_cast<float2 *>(g.tab), g.T, g.t0, g.Hg, g.Wg,
                                                 g.pt, g.py, g.px, theta);
    return cudaGetLastError();
}

cudaError_t launch_scan(const KGeom &g, int d, const float *S_in, const float *z_in, float *S_out,
                        float *z_out, cudaStream_t s) {
    const int E = d * d + d;
    dim3 grid((E + 255) / 256, g.BH);
    scan_kernel<<<grid, 256, 0, s>>>(g, d, S_in, z_in, S_out, z_out);
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

// Raise the dynamic shared-memory limit of a kernel once per device (one cache
// per kernel: the template parameter is the kernel itself, not its type).
template <auto Kernel>
static cudaError_t set_smem(int bytes) {
    static bool done[64] = {false};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && done[dev]) return cudaSuccess;
    e = cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && dev >= 0 && dev < 64) done[dev] = true;
    return e;
}

cudaError_t launch_partial_tc(const KGeom &g, int d, const CUtensorMap &mk, const CUtensorMap &mv,
                              cudaStream_t s) {
    int *wd = watchdog_ptr();
    if (wd == nullptr) return cudaErrorInvalidDevice;
    dim3 grid(g.cpb, g.nblk, g.BH);
    cudaError_t e;
    if (d == 32) {
        auto k = partial_tc_kernel<32, 4, 6, 6>;
        constexpr int smem = partial_tc_smem_bytes<32>();
        if ((e = set_smem<partial_tc_kernel<32, 4, 6, 6>>(smem)) != cudaSuccess) return e;
        k<<<grid, 160, smem, s>>>(mk, mv, g, wd);
    } else {
        auto k = partial_tc_kernel<64, 8, 12, 12>;
        constexpr int smem = partial_tc_smem_bytes<64>();
        if ((e = set_smem<partial_tc_kernel<64, 8, 12, 12>>(smem)) != cudaSuccess) return e;
        k<<<grid, 160, smem, s>>>(mk, mv, g, wd);
    }
    return cudaGetLastError();
}

cudaError_t launch_output_tc(const KGeom &g, int d, const CUtensorMap &mq, const CUtensorMap &mo,
                             void *o, cudaStream_t s) {
    int *wd = watchdog_ptr();
    if (wd == nullptr) return cudaErrorInvalidDevice;
    dim3 grid(g.qcpb, g.nblk, g.BH);
    cudaError_t e;
    __nv_bfloat16 *ob = static_cast<__nv_bfloat16 *>(o);
    if (d == 32) {
        auto k = output_tc_kernel<32, 4, 6, 6>;
        constexpr int smem = output_tc_smem_bytes<32>();
        if ((e = set_smem<output_tc_kernel<32, 4, 6, 6>>(smem)) != cudaSuccess) return e;
        k<<<grid, 160, smem, s>>>(mq, mo, g, ob, wd);
    } else {
        auto k = output_tc_kernel<64, 8, 12, 12>;
        constexpr int smem = output_tc_smem_bytes<64>();
        if ((e = set_smem<output_tc_kernel<64, 8, 12, 12>>(smem)) != cudaSuccess) return e;
        k<<<grid, 160, smem, s>>>(mq, mo, g, ob, wd);
    }
    return cudaGetLastError();
}

}  // namespace blin
