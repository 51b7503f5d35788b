// amk_probe.cu -- the read ceiling of the decode kernel's weight stream:
// the same bulk copies (cp.async.bulk into a shared-memory ring of stages on
// mbarriers, evict-first L2 policy, one CTA per SM) with nothing consuming
// them, over a buffer larger than L2.  The roofline of the decode step is
// reported against this beside the copy bandwidth (which counts read and
// write bytes): the step itself only reads.
#include <cuda_runtime.h>

#include "amk_kernel_body.cuh"

namespace amk {
namespace {

// CTA b streams bytes [b * per_cta, (b + 1) * per_cta) of buf in stage-sized
// copies, `stages` of them in flight.  Every wait is bounded; on expiry the
// CTA stops issuing and writes 1 to fail[b].
__global__ void __launch_bounds__(32, 1)
amk_read_probe_kernel(const uint8_t *buf, uint64_t per_cta, int stage_bytes, int stages,
                      unsigned int *fail)
{
    extern __shared__ __align__(1024) uint8_t smem[];
    if (threadIdx.x != 0)
        return;
    const uint32_t ring = smem_u32(smem);
    const uint32_t bars = ring + (uint32_t)(stages * stage_bytes);
    for (int i = 0; i < stages; ++i)
        mbar_init(bars + 8 * i, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    const uint64_t pol = evict_first_policy();
    const uint8_t *src = buf + (uint64_t)blockIdx.x * per_cta;
    const uint32_t n = (uint32_t)(per_cta / (uint64_t)stage_bytes);
    uint32_t k = 0;
    bool bad = false;
    for (; k < n && !bad; ++k) {
        const int st = (int)(k % (uint32_t)stages);
        if (k >= (uint32_t)stages) {
            const uint32_t par = ((k / stages) - 1) & 1;
            const uint64_t t0 = gtimer();
            while (!mbar_try_wait(bars + 8 * st, par))
                if (gtimer() - t0 > 1000000000ull) {  // 1 s
                    bad = true;
                    break;
                }
            if (bad)
                break;
        }
        mbar_arrive_expect_tx(bars + 8 * st, (uint32_t)stage_bytes);
        bulk_g2s(ring + (uint32_t)(st * stage_bytes), src + (uint64_t)k * stage_bytes,
                 (uint32_t)stage_bytes, bars + 8 * st, pol);
    }
    // drain: every copy issued lands before the CTA exits
    const uint32_t first = k > (uint32_t)stages ? k - stages : 0;
    for (uint32_t j = first; j < k; ++j) {
        const uint64_t t0 = gtimer();
        while (!mbar_try_wait(bars + 8 * (j % stages), (j / stages) & 1))
            if (gtimer() - t0 > 1000000000ull) {
                bad = true;
                break;
            }
    }
    if (bad)
        fail[blockIdx.x] = 1u;
}

}  // namespace
}  // namespace amk

// bytes / second of the stream over `bytes` of the device buffer `buf` (at
// least 1 GiB, larger than L2) on n_sms CTAs, with `stages` copies of
// stage_bytes in flight per SM, best of `reps` timed launches after one
// warm-up launch, on `stream`.
extern "C" int amk_read_ceiling(const void *buf, int64_t bytes, int n_sms, int stage_bytes,
                                int stages, int reps, void *stream, double *gbs)
{
    if (!buf || !gbs || bytes < (1ll << 30) || n_sms < 1 || stages < 1 || stages > 16 ||
        stage_bytes < 1024 || stage_bytes % 16 || reps < 1 ||
        (int64_t)stages * stage_bytes + 8 * stages > 227 * 1024)
        return amk_set_error(AMK_ERR_INVALID_ARG, "amk_read_ceiling: bad argument");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const uint64_t per_cta = (uint64_t)bytes / (uint64_t)n_sms / (uint64_t)stage_bytes *
                             (uint64_t)stage_bytes;
    const int smem = stages * stage_bytes + 8 * stages;
    unsigned int *fail = nullptr;
    cudaEvent_t a = nullptr, b = nullptr;
    cudaError_t e = cudaFuncSetAttribute(amk::amk_read_probe_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess)
        e = cudaMalloc(&fail, sizeof(unsigned int) * (size_t)n_sms);
    if (e == cudaSuccess)
        e = cudaMemsetAsync(fail, 0, sizeof(unsigned int) * (size_t)n_sms, st);
    if (e == cudaSuccess)
        e = cudaEventCreate(&a);
    if (e == cudaSuccess)
        e = cudaEventCreate(&b);
    double best = 0.0;
    for (int r = 0; e == cudaSuccess && r <= reps; ++r) {
        cudaEventRecord(a, st);
        amk::amk_read_probe_kernel<<<n_sms, 32, smem, st>>>(
            static_cast<const uint8_t *>(buf), per_cta, stage_bytes, stages, fail);
        cudaEventRecord(b, st);
        e = cudaEventSynchronize(b);
        float ms = 0.f;
        if (e == cudaSuccess)
            e = cudaEventElapsedTime(&ms, a, b);
        if (e == cudaSuccess && r > 0 && ms > 0.f)
            best = std::max(best, (double)per_cta * n_sms / (ms * 1e-3));
    }
    unsigned int f = 0;
    if (e == cudaSuccess) {
        for (int i = 0; i < n_sms && e == cudaSuccess; ++i) {
            unsigned int v = 0;
            e = cudaMemcpy(&v, fail + i, sizeof v, cudaMemcpyDeviceToHost);
            f |= v;
        }
    }
    if (a)
        cudaEventDestroy(a);
    if (b)
        cudaEventDestroy(b);
    if (fail)
        cudaFree(fail);
    if (e != cudaSuccess)
        return amk_set_error(AMK_ERR_CUDA, "amk_read_ceiling: %s", cudaGetErrorString(e));
    if (f)
        return amk_set_error(AMK_ERR_TIMEOUT, "amk_read_ceiling: a copy did not land in time");
    *gbs = best / 1e9;
    return AMK_OK;
}
