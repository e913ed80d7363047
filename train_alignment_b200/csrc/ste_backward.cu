// Straight-through backward of the weight fake-quant ([QUADS-fr §2.2.A]:
// the trainer's weights see the rollout's NVFP4 grid in the forward pass; the
// gradient passes through the rounding unchanged):
//   grad_w = grad_wfq                       (accumulate = 0)
//   grad_w = bf16(fp32(grad_w + grad_wfq))  (accumulate = 1)
// HBM-bound: 6 bytes per element with accumulation.
#include "common.cuh"

namespace quads {
namespace {

constexpr int kThreads = 256;

int ste_grid(int64_t work) {
  int64_t g = ceil_div(work, int64_t(kThreads));
  const int64_t cap = static_cast<int64_t>(num_sms()) * 8;
  return static_cast<int>(g > cap ? cap : (g < 1 ? 1 : g));
}

// Each thread keeps kSteUnroll 16-byte vectors of both inputs in flight per
// iteration of a grid-stride loop.
constexpr int kSteUnroll = 2;

__device__ __forceinline__ uint4 ste_add(uint4 a, uint4 b) {
  uint32_t* pa = reinterpret_cast<uint32_t*>(&a);
  const uint32_t* pb = reinterpret_cast<const uint32_t*>(&b);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float lo = __fadd_rn(bf16_bits_to_float(pa[j] & 0xFFFFu), bf16_bits_to_float(pb[j] & 0xFFFFu));
    const float hi = __fadd_rn(bf16_bits_to_float(pa[j] >> 16), bf16_bits_to_float(pb[j] >> 16));
    pa[j] = pack_bf16x2(lo, hi);
  }
  return a;
}

__global__ void __launch_bounds__(kThreads) ste_backward_kernel(const uint16_t* __restrict__ gfq,
                                                                uint16_t* __restrict__ gw, int64_t n, int accumulate) {
  const int64_t nv = n / 8;
  const int64_t nth = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const uint4* src = reinterpret_cast<const uint4*>(gfq);
  uint4* dst = reinterpret_cast<uint4*>(gw);
  int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (; i + (kSteUnroll - 1) * nth < nv; i += kSteUnroll * nth) {
    uint4 a[kSteUnroll], b[kSteUnroll];
#pragma unroll
    for (int u = 0; u < kSteUnroll; ++u) a[u] = __ldg(src + i + u * nth);
    if (accumulate) {
#pragma unroll
      for (int u = 0; u < kSteUnroll; ++u) b[u] = dst[i + u * nth];
#pragma unroll
      for (int u = 0; u < kSteUnroll; ++u) a[u] = ste_add(a[u], b[u]);
    }
#pragma unroll
    for (int u = 0; u < kSteUnroll; ++u) dst[i + u * nth] = a[u];
  }
  for (; i < nv; i += nth) {
    uint4 a = __ldg(src + i);
    if (accumulate) a = ste_add(a, dst[i]);
    dst[i] = a;
  }
  // tail (n % 8 elements) handled by the first thread
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    for (int64_t i = nv * 8; i < n; ++i) {
      if (accumulate)
        gw[i] = static_cast<uint16_t>(
            float_to_bf16_bits(__fadd_rn(bf16_bits_to_float(gfq[i]), bf16_bits_to_float(gw[i]))));
      else
        gw[i] = gfq[i];
    }
  }
}

}  // namespace
}  // namespace quads

using namespace quads;

extern "C" {

int quads_fakequant_weight_ste_backward(const uint16_t* grad_wfq, uint16_t* grad_w, int64_t n, int accumulate,
                                        quads_stream_t stream) {
  clear_error();
  QUADS_REQUIRE(n >= 0, QUADS_ERR_INVALID_ARG, "n must be >= 0");
  if (n == 0) return QUADS_OK;
  QUADS_REQUIRE(grad_wfq && grad_w && aligned(grad_wfq, 16) && aligned(grad_w, 16), QUADS_ERR_INVALID_ARG,
                "gradients must be non-null and 16-byte aligned");
  ste_backward_kernel<<<ste_grid(ceil_div(ceil_div(n, 8), int64_t(kSteUnroll))), kThreads, 0, stream>>>(
      grad_wfq, grad_w, n, accumulate);
  count_launches(1);
  return check_launch("ste_backward_kernel");
}

}  // extern "C"
