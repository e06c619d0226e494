// middle_bf16_f32.cu -- the middle of bf16 passes with float32 Q/K/V/G/O (shapes the row-gather attention does not take).
#include "middle.cuh"

namespace atomenc {
namespace host {
template void launch_middle<__nv_bfloat16, float>(PassCtx<__nv_bfloat16> &);
}  // namespace host
}  // namespace atomenc
