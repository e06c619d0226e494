// pass_f32.cu -- the launch sequence of float32 passes.
#include "pass.cuh"

namespace atomenc {
namespace host {
template int launch_all<float>(const Plan &, const atomenc_inputs *, const atomenc_params *, float, int64_t, const atomenc_outputs *, unsigned char *, cudaStream_t, Hooks &, int, unsigned char *);
}  // namespace host
}  // namespace atomenc
