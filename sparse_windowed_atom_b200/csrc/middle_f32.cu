// middle_f32.cu -- the middle of float32 passes.
#include "middle.cuh"

namespace atomenc {
namespace host {
template void launch_middle<float, float>(PassCtx<float> &);
}  // namespace host
}  // namespace atomenc
