// The discretisation-step prologue of the fused scan: dt <- clamp(softplus(dt + dt_bias)).
//
// In the Mamba-2 block the step dt of every (token, head) is a projection of the input passed
// through a softplus after a per-head bias, then clamped (mohakchugh.is-a.dev "Mamba-2",
// Architecture: Multi-Head SSM; the selection mechanism makes dt input-dependent).  The kernel
// writes the dt the scan uses into the workspace; every later kernel reads that.  HBM-bound
// elementwise pass, one float4 of a row per thread.
#include "common.cuh"

namespace ssd {
namespace {

__global__ void dt_prologue_kernel(const float *__restrict__ dt, const float *__restrict__ bias,
                                   float *__restrict__ out, int64_t n, int H, bool softplus,
                                   bool clamp, float lo, float hi)
{
    const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (i >= n) return;
    out[i] = dt_transform(dt[i], bias, (int)(i % H), softplus, clamp, lo, hi);
}

}  // namespace

cudaError_t launch_dt_prologue(const float *dt, const float *bias, float *dt_out, int64_t nrows,
                               int H, bool softplus, bool clamp, float lo, float hi,
                               cudaStream_t st)
{
    const int64_t n = nrows * H;
    if (n == 0) return cudaSuccess;
    dt_prologue_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(dt, bias, dt_out, n, H,
                                                                   softplus, clamp, lo, hi);
    return cudaGetLastError();
}

}  // namespace ssd
