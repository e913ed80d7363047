// Device helpers shared by the TRACE replay kernels (full record and the
// compact rounding-direction record).
#pragma once

#include "common.cuh"

namespace quads {

// Replayed operand on the compensation channels of one 512-column pass of a
// row: x_hat[c] = bf16(fp32(deq(code) + r)) for the pass's channel slots
// [slo, shi) (valid channels ascend, slot j taken by lane j % 32).  Each
// element's code and block scale come by shuffles from the lane that owns
// its 16-element block (q of every lane of the warp); called by all 32
// lanes after the pass's block stores.
__device__ __forceinline__ void replay_channel_pass(const QCore& q, float g, int p, int slo, int shi,
                                                    const int32_t* chan_s, const uint16_t* resid_row,
                                                    uint16_t* x_hat_row) {
  const int lane = threadIdx.x & 31;
  __syncwarp();
  for (int j0 = slo; j0 < shi; j0 += 32) {               // warp-uniform
    const int j = j0 + lane;
    const bool act = j < shi;
    const int c = act ? chan_s[j] : 512 * p;
    const int src = (c - 512 * p) >> 4, bit = c & 15;
    const uint32_t cl = __shfl_sync(0xffffffffu, q.lo, src);
    const uint32_t ch = __shfl_sync(0xffffffffu, q.hi, src);
    const float sv = __shfl_sync(0xffffffffu, q.sv, src);
    if (act) {
      const uint32_t code = (((bit < 8) ? cl : ch) >> (4 * (bit & 7))) & 15u;
      const float v = __fadd_rn(deq_f32(code, sv, g), bf16_bits_to_float(resid_row[j]));
      x_hat_row[c] = static_cast<uint16_t>(float_to_bf16_bits(v));
    }
  }
  __syncwarp();
}

}  // namespace quads
