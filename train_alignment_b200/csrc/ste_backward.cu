// Straight-through backward of the weight fake-quant ([QUADS-fr §2.2.A]:
// the trainer's weights see the rollout's NVFP4 grid in the forward pass; the
// gradient passes through the rounding unchanged):
//   grad_w = grad_wfq                       (accumulate = 0)
//   grad_w = bf16(fp32(grad_w + grad_wfq))  (accumulate = 1)
// HBM-bound: 6 bytes per element with accumulation.
#include "common.cuh"

namespace quads {
namespace {

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

// One CTA per SM (all SMs, or the SM budget), streaming through shared
// memory: the loads are bulk copies of one 16 KB chunk of each input per
// stage into a ring of six stages; sixteen arithmetic warps each add their
// own slice of a stage and store the sum with coalesced 16-byte stores.  The
// shared-memory request keeps a second CTA off the SM, so that under an SM
// budget the rollout's persistent GEMMs keep the other SMs to themselves.
constexpr int kTmaIssuers = 1;                 // loading warps per input (stages alternate between them)
constexpr int kTmaConsumerWarps = 16;
constexpr int kTmaThreads = 64 * kTmaIssuers + 32 * kTmaConsumerWarps;   // loading warps, then arithmetic warps
constexpr int kTmaChunk = 16384;               // bytes of each input per stage
constexpr int kTmaStages = 6;
static_assert(kTmaStages % kTmaIssuers == 0, "each stage keeps one loading warp per input");
static_assert(kTmaChunk % (16 * 32 * kTmaConsumerWarps) == 0, "whole vectors per lane in a full stage");
constexpr int kTmaSmem = kTmaStages * 2 * kTmaChunk + 3 * kTmaStages * 8 + 16;
constexpr uint64_t kTmaTimeoutNs = 4000000000ull;
constexpr uint64_t kTmaDrainNs = 500000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t gtimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void bar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ bool bar_test(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait for the phase of the given parity; false when the limit
// expired (recorded in *status) or another role of the CTA gave up.
__device__ __forceinline__ bool bar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                         unsigned int* status, uint64_t limit_ns) {
  if (bar_test(bar, parity)) return true;
  const uint64_t t0 = gtimer();
  while (true) {
    if (bar_test(bar, parity)) return true;
    if (abort_flag != nullptr && *abort_flag) return false;
    if (gtimer() - t0 > limit_ns) {
      if (abort_flag != nullptr) *abort_flag = 1;
      if (status != nullptr) atomicOr(status, 1u);
      return false;
    }
  }
}
__device__ __forceinline__ void bulk_copy_in(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// nv 16-byte vectors (8 elements each); the n % 8 tail is done by the caller's
// tail kernel.  Chunk c (kTmaChunk bytes of each input) goes to CTA c % grid.
__global__ void __launch_bounds__(kTmaThreads, 1)
    ste_backward_tma_kernel(const uint16_t* __restrict__ gfq, uint16_t* __restrict__ gw, int64_t nv, int accumulate,
                            unsigned int* status) {
  extern __shared__ __align__(16) uint8_t ring[];
  __shared__ int abort_flag;
  const uint32_t base = smem_u32(ring);
  const uint32_t bar0 = base + kTmaStages * 2 * kTmaChunk;
  auto full_bar = [&](int input, int s) { return bar0 + 8u * (input * kTmaStages + s); };
  auto empty_bar = [&](int s) { return bar0 + 8u * (2 * kTmaStages + s); };
  if (threadIdx.x == 0) {
    for (int s = 0; s < kTmaStages; ++s) {
      bar_init(full_bar(0, s), 1);
      bar_init(full_bar(1, s), 1);
      bar_init(empty_bar(s), kTmaConsumerWarps);
    }
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  volatile int* const abort_p = &abort_flag;
  constexpr int64_t kVpc = kTmaChunk / 16;      // vectors per chunk
  const int64_t nchunks = (nv + kVpc - 1) / kVpc;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp < 2 * kTmaIssuers) {
    // ---------------------------------------------------------- loads
    const int input = warp & 1, sub = warp >> 1;
    if (lane != 0 || (input == 1 && !accumulate)) return;
    const uint8_t* src = reinterpret_cast<const uint8_t*>(input == 0 ? gfq : gw);
    int it = 0, last = -1;
    bool ok = true;
    for (int64_t c = blockIdx.x; c < nchunks; c += gridDim.x, ++it) {
      if (it % kTmaIssuers != sub) continue;
      const int s = it % kTmaStages;
      if (!bar_wait(empty_bar(s), ((it / kTmaStages) & 1) ^ 1u, abort_p, status, kTmaTimeoutNs)) {
        ok = false;
        break;
      }
      const int64_t nvec = nv - c * kVpc < kVpc ? nv - c * kVpc : kVpc;
      bulk_copy_in(base + (2 * s + input) * kTmaChunk, src + c * kTmaChunk, static_cast<uint32_t>(nvec * 16),
                   full_bar(input, s));
      last = it;
    }
    if (!ok)   // this warp's copies in flight land before the CTA exits
      for (int i = (last >= kTmaStages ? last - kTmaStages + 1 : 0); i <= last; ++i)
        if (i % kTmaIssuers == sub)
          bar_wait(full_bar(input, i % kTmaStages), (i / kTmaStages) & 1, nullptr, nullptr, kTmaDrainNs);
    return;
  }
  // ---------------------------------------------------------- arithmetic
  // Warp w of the arithmetic warps takes its own slice of every stage: lane
  // 0 waits for the stage, the warp adds and stores its vectors, and lane 0
  // releases the stage (the empty barrier counts one arrival per warp).
  const int cw = warp - 2 * kTmaIssuers;
  constexpr int kPerWarp = kTmaChunk / 16 / kTmaConsumerWarps;   // vectors of a full stage per warp
  uint4* dst = reinterpret_cast<uint4*>(gw);
  int it = 0;
  for (int64_t c = blockIdx.x; c < nchunks; c += gridDim.x, ++it) {
    const int s = it % kTmaStages;
    const uint32_t ph = (it / kTmaStages) & 1;
    int ok = 1;
    if (lane == 0) {
      ok = bar_wait(full_bar(0, s), ph, abort_p, status, kTmaTimeoutNs) ? 1 : 0;
      if (ok && accumulate) ok = bar_wait(full_bar(1, s), ph, abort_p, status, kTmaTimeoutNs) ? 1 : 0;
    }
    if (!__shfl_sync(0xffffffffu, ok, 0)) break;
    const int64_t nvec = nv - c * kVpc < kVpc ? nv - c * kVpc : kVpc;
    const uint32_t sa = base + 2 * s * kTmaChunk;
    const int v0 = cw * kPerWarp;
    if (nvec == kVpc) {
      uint4 a[kPerWarp / 32];
#pragma unroll
      for (int u = 0; u < kPerWarp / 32; ++u) a[u] = lds128(sa + 16 * (v0 + u * 32 + lane));
      if (accumulate) {
#pragma unroll
        for (int u = 0; u < kPerWarp / 32; ++u) a[u] = ste_add(a[u], lds128(sa + kTmaChunk + 16 * (v0 + u * 32 + lane)));
      }
#pragma unroll
      for (int u = 0; u < kPerWarp / 32; ++u) dst[c * kVpc + v0 + u * 32 + lane] = a[u];
    } else {
      for (int v = v0 + lane; v < v0 + kPerWarp && v < nvec; v += 32) {
        uint4 a = lds128(sa + 16 * v);
        if (accumulate) a = ste_add(a, lds128(sa + kTmaChunk + 16 * v));
        dst[c * kVpc + v] = a;
      }
    }
    __syncwarp();
    if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(empty_bar(s)) : "memory");
  }
}

__global__ void ste_backward_tail_kernel(const uint16_t* __restrict__ gfq, uint16_t* __restrict__ gw, int64_t from,
                                         int64_t n, int accumulate) {
  for (int64_t i = from + threadIdx.x; i < n; i += blockDim.x) {
    if (accumulate)
      gw[i] = static_cast<uint16_t>(
          float_to_bf16_bits(__fadd_rn(bf16_bits_to_float(gfq[i]), bf16_bits_to_float(gw[i]))));
    else
      gw[i] = gfq[i];
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
  if (cudaFuncSetAttribute(ste_backward_tma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kTmaSmem) !=
      cudaSuccess)
    return set_error(QUADS_ERR_CUDA, "cannot reserve shared memory for the STE backward");
  const int64_t nv = n / 8;
  int launches = 0;
  if (nv > 0) {
    const int64_t nchunks = ceil_div(nv, int64_t(kTmaChunk / 16));
    const int grid = static_cast<int>(nchunks < grid_sms() ? nchunks : grid_sms());
    ste_backward_tma_kernel<<<grid, kTmaThreads, kTmaSmem, stream>>>(grad_wfq, grad_w, nv, accumulate,
                                                                     wait_status_word());
    ++launches;
  }
  if (nv * 8 < n) {
    ste_backward_tail_kernel<<<1, 32, 0, stream>>>(grad_wfq, grad_w, nv * 8, n, accumulate);
    ++launches;
  }
  count_launches(launches);
  return check_launch("ste_backward_tma_kernel");
}

}  // extern "C"
