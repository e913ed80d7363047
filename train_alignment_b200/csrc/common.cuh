// Shared host and device helpers of libquads (internal; not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "quads.h"

namespace quads {

// ------------------------------------------------------------------ host side

int set_error(int code, const char* fmt, ...);
// Grid for a persistent grid-stride kernel: min(work items / per_block,
// resident blocks per SM x SMs).
int persistent_grid(const void* kernel, int threads, size_t smem, int64_t work_blocks);
void clear_error();
void count_launches(uint64_t n);
int num_sms();
// The SM budget set by quads_set_sm_budget (0: none, or a budget of at least
// the device's SM count), and the SMs a persistent grid may use.
int sm_budget();
int grid_sms();
// Device address of the word in which bounded device-side waits record a
// timeout (read and cleared by quads_device_status), or null.
unsigned int* wait_status_word();

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

// Division of n < 2^31 by a fixed d >= 1 with a multiply-high and a shift
// (the round-up multiplier: s = ceil(log2 d), m = floor(2^32 (2^s - d) / d) + 1,
// n / d = (umulhi(n, m) + n) >> s).
struct FastDiv {
  uint32_t d, m, s;
};
inline FastDiv make_fastdiv(uint32_t d) {
  uint32_t s = 0;
  while ((uint64_t(1) << s) < d) ++s;
  uint64_t m = ((uint64_t(1) << 32) * ((uint64_t(1) << s) - d)) / d + 1;
  return FastDiv{d, static_cast<uint32_t>(m), s};
}
__device__ __forceinline__ uint32_t fast_div(uint32_t n, const FastDiv& f) { return (__umulhi(n, f.m) + n) >> f.s; }

// ---------------------------------------------------------------- device side


constexpr float kNvfp4Range = 2688.0f;   // 6 * 448

__device__ __forceinline__ float bf16_bits_to_float(uint32_t b) { return __uint_as_float(b << 16); }

__device__ __forceinline__ uint32_t float_to_bf16_bits(float f) {
  return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(f)));
}

// Two floats -> packed BF16 pair (lo in the low half), round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
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

// ---- packed helpers (two fp32 in a 64-bit register: element 0 in the low half)

__device__ __forceinline__ uint64_t pack_f32x2(float lo, float hi) {
  return (static_cast<uint64_t>(__float_as_uint(hi)) << 32) | __float_as_uint(lo);
}
__device__ __forceinline__ float lo_f32(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v)); }
__device__ __forceinline__ float hi_f32(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v >> 32)); }
// Two IEEE round-to-nearest fp32 products in one instruction.
__device__ __forceinline__ uint64_t fmul2_rn(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
// A word of two BF16 values -> the two values as fp32 (exact).
__device__ __forceinline__ uint64_t bf16x2_to_f32x2(uint32_t w) {
  return (static_cast<uint64_t>(w & 0xFFFF0000u) << 32) | (w << 16);
}
// Two floats -> BF16 pair, lo in the low half (round to nearest even), one instruction.
__device__ __forceinline__ uint32_t f32x2_to_bf16x2(uint64_t v) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi_f32(v)), "f"(lo_f32(v)));
  return r;
}

// Eight packed fp32 pairs (elements 2i, 2i+1 in y[i]) -> eight E2M1 codes,
// element i in nibble i (nearest-even, saturating, sign kept).
__device__ __forceinline__ uint32_t e2m1x8_from_pairs(const uint64_t* y) {
  float v[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = lo_f32(y[i]);
    v[2 * i + 1] = hi_f32(y[i]);
  }
  return e2m1x8_from_float(v);
}

// Eight E2M1 codes (nibble i = element i) -> four f16x2 values (exact).
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t codes, uint32_t (&h)[4]) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
      : "r"(codes));
}
// f16x2 product (exact here: both factors carry few significant bits).
__device__ __forceinline__ uint32_t hmul2_rn(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
// f16x2 -> two fp32 (exact).
__device__ __forceinline__ uint64_t f16x2_to_f32x2(uint32_t h) {
  float lo, hi;
  asm("{\n\t.reg .f16 l, u;\n\tmov.b32 {l, u}, %2;\n\tcvt.f32.f16 %0, l;\n\tcvt.f32.f16 %1, u;\n\t}"
      : "=f"(lo), "=f"(hi)
      : "r"(h));
  return pack_f32x2(lo, hi);
}
// An E4M3 scale value (exactly representable in f16) as an f16x2 pair.
__device__ __forceinline__ uint32_t f16x2_splat(float v) {
  uint32_t r;
  asm("{\n\t.reg .f16 t;\n\tcvt.rn.f16.f32 t, %1;\n\tmov.b32 %0, {t, t};\n\t}" : "=r"(r) : "f"(v));
  return r;
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
  FastDiv uniform;           // rows per group when off_smem is null
  __device__ __forceinline__ int of(int64_t row) const {
    if (off_smem == nullptr) {
      if (n == 1) return 0;
      return static_cast<int>(fast_div(static_cast<uint32_t>(row), uniform));
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

// One quantized block: codes (nibble i = element i), E4M3 scale and its value.
struct QCore {
  uint32_t lo, hi, scale;
  float sv;
};

// Per-group constants of the block-scale computation: the per-tensor scale g,
// d = fp32(6 g), rd = fp32(1 / d) when the division below may use it (0
// otherwise), and optionally a table tab[s] = {S, fp32(1 / S)} with
// S = fp32(val(s) g) for every E4M3 code s in [0, 128).
struct QConsts {
  float g, d, rd;
  const float2* tab;
};

__device__ __forceinline__ QConsts make_qconsts(float g, const float2* tab = nullptr) {
  QConsts c;
  c.g = g;
  c.d = __fmul_rn(6.0f, g);
  c.rd = (c.d >= 0x1p-60f) ? __frcp_rn(c.d) : 0.0f;
  c.tab = tab;
  return c;
}

// Entry s of the {S, 1/S} table of a group.
__device__ __forceinline__ float2 scale_table_entry(uint32_t s, float g) {
  const float S = __fmul_rn(e4m3_value(s), g);
  return make_float2(S, S != 0.0f ? __frcp_rn(S) : 0.0f);
}

// fp32(amax / d), correctly rounded.  With rd = fp32(1/d), q = fp32(amax rd)
// is within one ulp of the quotient, the remainder amax - d q is exact in one
// FMA, and fp32(q + rem rd) is the correctly rounded quotient (Markstein's
// theorem; P. Markstein, IBM J. Res. Develop. 34(1), 1990).  rd is set only
// for d >= 2^-60, where every remainder that can change an E4M3 scale stays a
// normal number; smaller d takes the full division.
__device__ __forceinline__ float block_ratio(float amax, const QConsts& c) {
  if (c.rd == 0.0f) return __fdiv_rn(amax, c.d);
  const float q = __fmul_rn(amax, c.rd);
  const float rem = __fmaf_rn(-c.d, q, amax);
  return __fmaf_rn(rem, c.rd, q);
}

// {val(s), val(s)} as an f16x2 pair (exact: E4M3 values are f16 values).
__device__ __forceinline__ uint32_t e4m3_splat_f16x2(uint32_t s) {
  uint32_t r;
  const uint16_t in = static_cast<uint16_t>(s | (s << 8));
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(in));
  return r;
}

// The quantizer on 16 BF16 values given as 8 packed words (element 2i in the
// low half of w[i]); same operations and rounding as quantize_block.
__device__ __forceinline__ QCore quant_core(const uint32_t (&w)[8], const QConsts& c) {
  // lane-wise max |.| of the pairs in one instruction each (the result's sign
  // bits, the XOR of the inputs', are cleared afterwards)
  uint32_t m = 0u;
#pragma unroll
  for (int i = 0; i < 8; ++i) asm("max.xorsign.abs.bf16x2 %0, %0, %1;" : "+r"(m) : "r"(w[i]));
  m &= 0x7FFF7FFFu;
  const float amax = bf16_bits_to_float(max(m & 0xFFFFu, m >> 16));
  uint32_t s = 0;
  if (c.g != 0.0f) s = e4m3_from_float(block_ratio(amax, c));
  QCore r;
  r.scale = s;
  r.sv = e4m3_value(s);
  float S, inv;
  if (c.tab != nullptr) {
    const float2 e = c.tab[s];
    S = e.x;
    inv = e.y;
  } else {
    S = __fmul_rn(r.sv, c.g);
    inv = (S != 0.0f) ? __frcp_rn(S) : 0.0f;
  }
  if (S == 0.0f) {
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      lo |= ((w[i] >> 15) & 1u) << (8 * i + 3) | ((w[i] >> 31) & 1u) << (8 * i + 7);
      hi |= ((w[4 + i] >> 15) & 1u) << (8 * i + 3) | ((w[4 + i] >> 31) & 1u) << (8 * i + 7);
    }
    r.lo = lo;
    r.hi = hi;
    return r;
  }
  const uint64_t inv2 = pack_f32x2(inv, inv);
  uint64_t y[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) y[i] = fmul2_rn(bf16x2_to_f32x2(w[i]), inv2);
  r.lo = e2m1x8_from_pairs(y);
  r.hi = e2m1x8_from_pairs(y + 4);
  return r;
}

__device__ __forceinline__ QCore quant_core(const uint32_t (&w)[8], float g) { return quant_core(w, make_qconsts(g)); }

// BF16 of the dequantized block: fp32(e2m1 * e4m3 * g) (fold) or the exact
// e2m1 * e4m3; the products e2m1 * e4m3 are exact in f16.
__device__ __forceinline__ void deq_block_bf16(const QCore& q, float g, int fold, uint32_t (&out)[8]) {
  uint32_t h[8];
  uint32_t h0[4], h1[4];
  e2m1x8_to_f16x2(q.lo, h0);
  e2m1x8_to_f16x2(q.hi, h1);
#pragma unroll
  for (int i = 0; i < 4; ++i) { h[i] = h0[i]; h[4 + i] = h1[i]; }
  const uint32_t sv2 = e4m3_splat_f16x2(q.scale);
  const uint64_t g2 = pack_f32x2(g, g);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    uint64_t f = f16x2_to_f32x2(hmul2_rn(h[i], sv2));
    if (fold) f = fmul2_rn(f, g2);
    out[i] = f32x2_to_bf16x2(f);
  }
}

}  // namespace quads
