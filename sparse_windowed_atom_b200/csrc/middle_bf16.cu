// middle_bf16.cu -- the middle of bf16 passes with bf16 Q/K/V/G/O.
#include "middle.cuh"

namespace atomenc {
namespace host {
template void launch_middle<__nv_bfloat16, __nv_bfloat16>(PassCtx<__nv_bfloat16> &);
}  // namespace host
}  // namespace atomenc
