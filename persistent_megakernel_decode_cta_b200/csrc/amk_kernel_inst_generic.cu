// amk_kernel_inst_generic.cu -- the generic kernel instance: every weight
// format and vector width dispatched at run time (models with odd row widths,
// or a bf16 tied head on int8 layers).
#include "amk_kernel_body.cuh"

namespace amk {
const void *amk_kernel_generic() { return reinterpret_cast<const void *>(amk_decode_kernel<0, 0, 1, 1>); }
}  // namespace amk
