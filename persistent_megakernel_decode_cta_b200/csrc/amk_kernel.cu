// amk_kernel.cu -- launch helpers of the persistent decode megakernel
// (the device code is in amk_kernel_body.cuh; its template instances are
// compiled by amk_kernel_inst_*.cu) and the Wdown packing kernel.
#include <cuda_runtime.h>
#include <stdint.h>

#include "amk_internal.h"

namespace amk {

// instance tables (amk_kernel_inst_*.cu), by attention lane width index e
// (lane width 1 << e, 16 for e >= 4)
const void *amk_kernel_q0_f0(int e);
const void *amk_kernel_q0_f1(int e);
const void *amk_kernel_q1_f0(int e);
const void *amk_kernel_q1_f1(int e);
const void *amk_kernel_q2_f0(int e);
const void *amk_kernel_generic();

// Wdown of one layer, [hidden][ffn] row-major, re-laid once per handle as
// 16-byte column groups, [ffn * esz / 16][hidden][16 B], so that a fused FFN
// slice's columns for a run of rows are contiguous: one thread per (column
// group, row), consecutive threads on consecutive rows (coalesced stores).
__global__ void amk_pack_down_kernel(const uint4 *wd, uint4 *out, int h, int ncg)
{
    const size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (size_t)h * ncg)
        return;
    const int row = (int)(idx % h), cg = (int)(idx / h);
    out[(size_t)cg * h + row] = wd[(size_t)row * ncg + cg];
}

// Host-visible launch helpers -------------------------------------------------
extern "C" int amk_kernel_smem_bytes(int ring_stages, int stage_bytes, int vec_floats)
{
    return ring_stages * stage_bytes + vec_floats * 4 + kConsumerWarps * kMaxTaskRows * 4 +
           (kPieces + 1) * kMaxStages * 8 + 16 * 4 + 64 * 4 + 2 * 8 + kPieceQueue * 16 +
           4 * (int)sizeof(TaskDesc);
}

namespace {
const void *kernel_for(int quant, int att_e, int generic, int fused)
{
    if (generic)
        return amk_kernel_generic();
    int e = 0;
    while (e < 4 && (1 << e) < att_e)
        ++e;
    if (quant == 2)  // int4 models never take the fused FFN level
        return amk_kernel_q2_f0(e);
    if (quant)
        return fused ? amk_kernel_q1_f1(e) : amk_kernel_q1_f0(e);
    return fused ? amk_kernel_q0_f1(e) : amk_kernel_q0_f0(e);
}
}  // namespace

extern "C" cudaError_t amk_kernel_configure(int smem_bytes, int quant, int att_e, int generic,
                                            int fused)
{
    return cudaFuncSetAttribute(kernel_for(quant, att_e, generic, fused),
                                cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
}

extern "C" cudaError_t amk_kernel_occupancy(int smem_bytes, int quant, int att_e, int generic,
                                            int fused, int *blocks_per_sm)
{
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(
        blocks_per_sm, kernel_for(quant, att_e, generic, fused), kThreads, smem_bytes);
}

extern "C" cudaError_t amk_pack_down(const void *wd, void *out, int h, int ffn, int esz,
                                     cudaStream_t stream)
{
    const int ncg = ffn * esz / 16;
    const size_t n = (size_t)h * ncg;
    amk_pack_down_kernel<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(
        static_cast<const uint4 *>(wd), static_cast<uint4 *>(out), h, ncg);
    return cudaGetLastError();
}

// An int4 matrix [rows][K / 2] with fp16 scales [rows][ceil(K / 128)], re-laid
// once per handle as rows of q4_row_bytes(K): the codes, the scales, zeros.
// One thread per 16-bit unit of the output (K / 2 is a multiple of 16).
__global__ void amk_pack_q4_kernel(const uint16_t *codes, const uint16_t *scales, uint16_t *out,
                                   int rows, int K)
{
    const int U = q4_row_bytes(K) / 2, cu = K / 4, ng = (K + kQ4Group - 1) / kQ4Group;
    const size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (size_t)rows * U)
        return;
    const int row = (int)(idx / U), u = (int)(idx % U);
    uint16_t v = 0;
    if (u < cu)
        v = codes[(size_t)row * cu + u];
    else if (u < cu + ng)
        v = scales[(size_t)row * ng + (u - cu)];
    out[idx] = v;
}

extern "C" cudaError_t amk_pack_q4(const void *codes, const void *scales, void *out, int rows,
                                   int K, cudaStream_t stream)
{
    const size_t n = (size_t)rows * (q4_row_bytes(K) / 2);
    amk_pack_q4_kernel<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(
        static_cast<const uint16_t *>(codes), static_cast<const uint16_t *>(scales),
        static_cast<uint16_t *>(out), rows, K);
    return cudaGetLastError();
}

extern "C" cudaError_t amk_kernel_launch(const KParams *p, int n_ctas, int smem_bytes,
                                         cudaStream_t stream)
{
    void *args[] = {const_cast<KParams *>(p)};
    return cudaLaunchCooperativeKernel(kernel_for(p->quant, p->att_e, p->generic, p->ffn_fused),
                                       dim3(n_ctas),
                                       dim3(kThreads), args, (size_t)smem_bytes, stream);
}

}  // namespace amk
