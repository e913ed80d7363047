// Shared host and device helpers of libquads (internal; not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "quads.h"

namespace quads {

// ------------------------------------------------------------------ host side

int set_error(int code, const char* fmt, ...);
void clear_error();
void count_launches(uint64_t n);
int num_sms();

// Returns QUADS_ERR_CUDA (with a message) if the last launch failed.
int check_launch(const char* what);

#define QUADS_REQUIRE(cond, code, ...)                 \
  do {                                                 \
    if (!(cond)) return ::quads::set_error((code), __VA_ARGS__); \
  } while (0)

#define QUADS_TRY(expr)               \
  do {                                \
    int _rc = (expr);                 \
    if (_rc != QUADS_OK) return _rc;  \
  } while (0)

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
__host__ __device__ inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Block-scale bytes for `rows` x K/16 scales.
__host__ __device__ inline int64_t scale_bytes(int64_t rows, int64_t K, int layout) {
  int64_t nkb = K / 16;
  if (layout == QUADS_SCALES_LINEAR) return rows * nkb;
  return ceil_div(rows, 128) * 128 * ceil_div(nkb, 4) * 4;
}

// ---------------------------------------------------------------- device side

constexpr float kNvfp4Range = 2688.0f;   // 6 * 448

__device__ __forceinline__ float bf16_bits_to_float(uint32_t b) { return __uint_as_float(b << 16); }

__device__ __forceinline__ uint32_t float_to_bf16_bits(float f) {
  return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(f)));
}

// Two floats -> packed BF16 pair (lo in the low half).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  return float_to_bf16_bits(lo) | (float_to_bf16_bits(hi) << 16);
}

// Value of an E4M3 (fn) scale code with the sign bit clear: 4 exponent bits
// (bias 7), 3 mantissa bits, exponent 0 subnormal (m * 2^-9).
__device__ __forceinline__ float e4m3_value(uint32_t c) {
  uint32_t e = (c >> 3) & 15u, m = c & 7u;
  if (e == 0) return static_cast<float>(m) * 0x1p-9f;
  return __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// Nearest-even, saturating conversion of a non-negative float to E4M3.
__device__ __forceinline__ uint32_t e4m3_from_float(float t) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(t));
  return r & 0xFFu;
}

// Eight floats -> eight E2M1 codes packed in 32 bits, element i in nibble i
// (nearest-even, saturating at +-6, sign kept).
__device__ __forceinline__ uint32_t e2m1x8_from_float(const float* v) {
  uint32_t out;
  asm("{\n\t"
      ".reg .b8 q0, q1, q2, q3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q3, %8, %7;\n\t"
      "mov.b32 %0, {q0, q1, q2, q3};\n\t"
      "}"
      : "=r"(out)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  return out;
}

// Value of a 4-bit E2M1 code: magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}.
__device__ __forceinline__ float e2m1_value(uint32_t c) {
  uint32_t m = c & 7u;
  float mag = (m < 4u) ? 0.5f * static_cast<float>(m)
                       : static_cast<float>((m & 1u) ? ((m == 7u) ? 6u : 3u) : ((m == 6u) ? 4u : 2u));
  return (c & 8u) ? -mag : mag;
}

// Byte offset of scale (row, kb) in the tiled layout with n_col_tiles tiles per row band.
__device__ __forceinline__ int64_t tiled_scale_offset(int64_t row, int64_t kb, int64_t n_col_tiles) {
  return ((row >> 7) * n_col_tiles + (kb >> 2)) * 512 + (row & 31) * 16 + ((row >> 5) & 3) * 4 + (kb & 3);
}

// Group of a row: explicit offsets (in shared memory) or uniform blocks of rows.
struct RowGroups {
  const int32_t* off_smem;   // n + 1 entries, or nullptr
  int n;
  int64_t uniform_rows;
  __device__ __forceinline__ int of(int64_t row) const {
    if (off_smem == nullptr) {
      if (n == 1) return 0;
      return static_cast<int>(row / uniform_rows);
    }
    int lo = 0, hi = n - 1;             // last i with off[i] <= row
    while (lo < hi) {
      int mid = (lo + hi + 1) >> 1;
      if (off_smem[mid] <= row) lo = mid; else hi = mid - 1;
    }
    return lo;
  }
};

// Load 16 BF16 values (32 bytes, 16-byte aligned) as raw bits.
__device__ __forceinline__ void load_bf16x16(const uint16_t* p, uint32_t (&w)[8]) {
  uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
  uint4 b = __ldg(reinterpret_cast<const uint4*>(p) + 1);
  w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
  w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
}

// One NVFP4 block: 16 values, their E4M3 scale and E2M1 codes under decode scale g.
struct QBlock {
  float x[16];
  uint32_t scale;       // E4M3 code
  float sv;             // its value
  uint32_t codes_lo;    // elements 0..7, nibble i = element i
  uint32_t codes_hi;    // elements 8..15
};

// Quantize one block of 16 floats (BF16-exact values) with decode scale g:
//   t = fp32(amax_b / fp32(6 g)), s = E4M3_RN_satfinite(t), S = fp32(val(s) g),
//   q_i = E2M1_RNE(fp32(x_i * fp32(1 / S))); S == 0 gives signed zeros.
__device__ __forceinline__ void quantize_block(QBlock& b, float g) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(b.x[i]));
  uint32_t s = 0;
  if (g != 0.0f) {
    float d = __fmul_rn(6.0f, g);
    float t = __fdiv_rn(amax, d);
    s = e4m3_from_float(t);
  }
  float sv = e4m3_value(s);
  float S = __fmul_rn(sv, g);
  b.scale = s;
  b.sv = sv;
  if (S == 0.0f) {
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      lo |= (__float_as_uint(b.x[i]) >> 31) << (4 * i + 3);
      hi |= (__float_as_uint(b.x[8 + i]) >> 31) << (4 * i + 3);
    }
    b.codes_lo = lo;
    b.codes_hi = hi;
    return;
  }
  float inv = __frcp_rn(S);
  float y[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) y[i] = __fmul_rn(b.x[i], inv);
  b.codes_lo = e2m1x8_from_float(y);
  b.codes_hi = e2m1x8_from_float(y + 8);
}

// Code of element i of a quantized block.
__device__ __forceinline__ uint32_t qblock_code(const QBlock& b, int i) {
  return ((i < 8 ? b.codes_lo >> (4 * i) : b.codes_hi >> (4 * (i - 8)))) & 15u;
}

// fp32(val(q) * val(s) * g) -- exact product of the first two, one rounding.
__device__ __forceinline__ float deq_f32(uint32_t code, float sv, float g) {
  return __fmul_rn(__fmul_rn(e2m1_value(code), sv), g);
}

}  // namespace quads
