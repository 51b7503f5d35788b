// amk_kernel_inst_i4_split.cu -- the kernel instances for packed int4 (W4A16)
// weights, one per attention lane width.  int4 models keep separate FFN
// levels (no fused int4 down projection), so there is no fused variant.
#include "amk_kernel_body.cuh"

namespace amk {
const void *amk_kernel_q2_f0(int e)
{
    switch (e) {
    case 0: return reinterpret_cast<const void *>(amk_decode_kernel<2, 1, 0, 0>);
    case 1: return reinterpret_cast<const void *>(amk_decode_kernel<2, 2, 0, 0>);
    case 2: return reinterpret_cast<const void *>(amk_decode_kernel<2, 4, 0, 0>);
    case 3: return reinterpret_cast<const void *>(amk_decode_kernel<2, 8, 0, 0>);
    default: return reinterpret_cast<const void *>(amk_decode_kernel<2, 16, 0, 0>);
    }
}
}  // namespace amk
