// amk_kernel_inst_i8_fused.cu -- the kernel instances for int8 (W8A16) weights with
// the fused FFN level, one per attention lane width.
#include "amk_kernel_body.cuh"

namespace amk {
const void *amk_kernel_q1_f1(int e)
{
    switch (e) {
    case 0: return reinterpret_cast<const void *>(amk_decode_kernel<1, 1, 0, 1>);
    case 1: return reinterpret_cast<const void *>(amk_decode_kernel<1, 2, 0, 1>);
    case 2: return reinterpret_cast<const void *>(amk_decode_kernel<1, 4, 0, 1>);
    case 3: return reinterpret_cast<const void *>(amk_decode_kernel<1, 8, 0, 1>);
    default: return reinterpret_cast<const void *>(amk_decode_kernel<1, 16, 0, 1>);
    }
}
}  // namespace amk
