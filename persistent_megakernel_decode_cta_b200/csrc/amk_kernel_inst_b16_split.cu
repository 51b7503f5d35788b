// amk_kernel_inst_b16_split.cu -- the kernel instances for bf16 weights with
// split FFN levels, one per attention lane width.
#include "amk_kernel_body.cuh"

namespace amk {
const void *amk_kernel_q0_f0(int e)
{
    switch (e) {
    case 0: return reinterpret_cast<const void *>(amk_decode_kernel<0, 1, 0, 0>);
    case 1: return reinterpret_cast<const void *>(amk_decode_kernel<0, 2, 0, 0>);
    case 2: return reinterpret_cast<const void *>(amk_decode_kernel<0, 4, 0, 0>);
    case 3: return reinterpret_cast<const void *>(amk_decode_kernel<0, 8, 0, 0>);
    default: return reinterpret_cast<const void *>(amk_decode_kernel<0, 16, 0, 0>);
    }
}
}  // namespace amk
