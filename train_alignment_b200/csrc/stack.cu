// The two operations that join MoE layers into a stack: the router
// projection of a layer's input and the residual connection.
//
// The pages' layers sit in a model whose other parts (attention, norms) the
// pages do not describe; the stack here is the plainest one the rest
// supports: x_{l+1} = x_l + MoE_l(x_l), router logits_l = x_l . W_r[l].
//
// router_logits_kernel: a 64-token x 64-expert output tile per 256-thread
// CTA, 4 x 4 outputs per thread, K staged through shared memory in chunks of
// 32; each output is an FP32 FMA chain over k in increasing order.
// residual_add_kernel: elementwise, 8 BF16 per thread and step.
#include "common.cuh"

namespace quads {
namespace {

constexpr int kTileT = 64, kTileE = 64, kChunk = 32;

__global__ void __launch_bounds__(256) router_logits_kernel(const uint16_t* __restrict__ x, int64_t T, int64_t H,
                                                            const float* __restrict__ w_r, int E,
                                                            float* __restrict__ logits) {
  __shared__ float xs[kChunk][kTileT + 1];      // [k][token]
  __shared__ float ws[kChunk][kTileE];          // [k][expert]
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kTileT;
  const int e0 = blockIdx.y * kTileE;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;   // 16 x 16 threads, 4 x 4 outputs each
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;
  for (int64_t k0 = 0; k0 < H; k0 += kChunk) {
    for (int i = threadIdx.x; i < kChunk * kTileT; i += blockDim.x) {
      const int kk = i % kChunk, tt = i / kChunk;
      const int64_t t = t0 + tt, k = k0 + kk;
      xs[kk][tt] = (t < T && k < H) ? bf16_bits_to_float(x[t * H + k]) : 0.0f;
    }
    for (int i = threadIdx.x; i < kChunk * kTileE; i += blockDim.x) {
      const int kk = i / kTileE, ee = i % kTileE;
      const int64_t k = k0 + kk;
      ws[kk][ee] = (k < H && e0 + ee < E) ? w_r[k * E + e0 + ee] : 0.0f;
    }
    __syncthreads();
    const int kn = static_cast<int>(H - k0 < kChunk ? H - k0 : kChunk);
    for (int kk = 0; kk < kn; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = xs[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = ws[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = __fmaf_rn(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t t = t0 + ty * 4 + i;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = e0 + tx * 4 + j;
      if (t < T && e < E) logits[t * E + e] = acc[i][j];
    }
  }
}

__global__ void __launch_bounds__(256) residual_add_kernel(const uint16_t* x, const uint16_t* y, int64_t n,
                                                           uint16_t* out) {
  const int64_t nv = n / 8;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nv;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint4 a = reinterpret_cast<const uint4*>(x)[i];      // plain loads: out may alias x or y
    const uint4 b = reinterpret_cast<const uint4*>(y)[i];
    const uint32_t* pa = reinterpret_cast<const uint32_t*>(&a);
    const uint32_t* pb = reinterpret_cast<const uint32_t*>(&b);
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
      o[j] = pack_bf16x2(__fadd_rn(bf16_bits_to_float(pa[j] & 0xFFFFu), bf16_bits_to_float(pb[j] & 0xFFFFu)),
                         __fadd_rn(bf16_bits_to_float(pa[j] >> 16), bf16_bits_to_float(pb[j] >> 16)));
    reinterpret_cast<uint4*>(out)[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// A few floats copied by the SMs (no copy engine, so a captured step's own
// small copies never queue behind host transfers on the copy engines).
__global__ void copy_f32_kernel(const float* src, float* dst, int64_t n) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    dst[i] = src[i];
}

}  // namespace
}  // namespace quads

using namespace quads;

extern "C" {

int quads_router_logits(const uint16_t* x, int64_t T, int64_t H, const float* w_r, int E, float* logits,
                        quads_stream_t stream) {
  clear_error();
  QUADS_REQUIRE(T >= 0 && H > 0, QUADS_ERR_INVALID_ARG, "T must be >= 0 and H > 0");
  QUADS_REQUIRE(E >= 1 && E <= 4096, QUADS_ERR_UNSUPPORTED_SHAPE, "E must be in [1, 4096]");
  if (T == 0) return QUADS_OK;
  QUADS_REQUIRE(x && w_r && logits, QUADS_ERR_INVALID_ARG, "null pointer");
  QUADS_REQUIRE(T < (int64_t(1) << 31) / kTileT * kTileT, QUADS_ERR_UNSUPPORTED_SHAPE, "T too large");
  const dim3 grid(static_cast<unsigned>(ceil_div(T, kTileT)), static_cast<unsigned>(ceil_div(E, kTileE)));
  router_logits_kernel<<<grid, 256, 0, stream>>>(x, T, H, w_r, E, logits);
  count_launches(1);
  return check_launch("router_logits_kernel");
}

int quads_residual_add(const uint16_t* x, const uint16_t* y, int64_t n, uint16_t* out, quads_stream_t stream) {
  clear_error();
  QUADS_REQUIRE(n >= 0 && n % 8 == 0, QUADS_ERR_INVALID_ARG, "n must be a non-negative multiple of 8");
  if (n == 0) return QUADS_OK;
  QUADS_REQUIRE(x && y && out && aligned(x, 16) && aligned(y, 16) && aligned(out, 16), QUADS_ERR_INVALID_ARG,
                "x, y and out must be non-null and 16-byte aligned");
  const int64_t want = ceil_div(n / 8, int64_t(256));
  const int grid = static_cast<int>(want < 4 * num_sms() ? want : 4 * num_sms());
  residual_add_kernel<<<grid, 256, 0, stream>>>(x, y, n, out);
  count_launches(1);
  return check_launch("residual_add_kernel");
}

int quads_copy_f32(const float* src, float* dst, int64_t n, quads_stream_t stream) {
  clear_error();
  QUADS_REQUIRE(n >= 0, QUADS_ERR_INVALID_ARG, "n must be >= 0");
  if (n == 0) return QUADS_OK;
  QUADS_REQUIRE(src && dst, QUADS_ERR_INVALID_ARG, "null pointer");
  const int64_t blocks = ceil_div(n, int64_t(256));
  copy_f32_kernel<<<static_cast<unsigned>(blocks < 1024 ? blocks : 1024), 256, 0, stream>>>(src, dst, n);
  count_launches(1);
  return check_launch("copy_f32_kernel");
}

}  // extern "C"
