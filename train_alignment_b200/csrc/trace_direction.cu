// Compact TRACE record: one rounding-direction bit per element in place of
// the 4-bit code, and the trainer's rounding guided by it.
//
// Method: [TRACE] "Fonctionnement, côté ingénierie" -- on a block-scaled FP4
// grid the rounding of each value is a discrete choice (up to the grid point
// above, or down to the one below); the trainer reads the rollout's record
// and uses it to make the same choice.  [TRACE] "L'idée centrale" -- the
// cache keeps the mantissa and the scale factors selectively, to save memory.
//
// For an element with block scale S = fp32(val(s) g) and y = fp32(x fp32(1/S)):
//   level(y) = index of the largest E2M1 level <= |y| (0 .. 7; 7 = 6.0);
//   rollout bit = 1 if its code's magnitude index is above level(y), else 0;
//   trainer code = sign(y_t) | min(level(y_t) + bit, 7).
// Blocks with S == 0 record 0 and replay signed zeros (the quantizer's rule).
// The trainer keeps the recorded block and per-tensor scales, so where both
// values lie between the same two levels the guided code is the rollout's.
//
// Both kernels: one warp per row, lane = 16-element block, 32 blocks per pass;
// HBM-bound streams (direction: 2 + 0.5 B read, 0.125 B written per element;
// replay: 2 + 0.125 B read, 2 (+ 0.5) B written).
#include "trace_common.cuh"

namespace quads {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxGroups = 1024;
constexpr int kMaxChan = 256;
// Up to this many groups, the {S, 1/S} pair of every E4M3 scale code of each
// group (S = fp32(val(s) g)) is tabulated in shared memory once per block
// instead of being computed (an E4M3 decode and a reciprocal) per block of
// 16 elements.
constexpr int kDirTabGroups = 16;

size_t dir_tab_bytes(int n_groups) {
  return n_groups <= kDirTabGroups ? static_cast<size_t>(n_groups) * 128 * sizeof(float2) : 0;
}

struct DirArgs {
  const uint16_t* x;          // rollout input (bits) or trainer input (replay)
  const uint8_t* codes;       // rollout codes (bits) or null
  const uint8_t* scales;
  int tiled;
  const float* g;
  const int32_t* group_off;
  int n_groups;
  FastDiv uniform;            // rows per group without group_off
  int64_t rows, K;
  uint8_t* bits;              // written (bits) / read (replay)
  // replay only
  const int32_t* chan;
  int n_chan;
  const uint16_t* resid;
  uint16_t* x_hat;
  uint8_t* codes_out;
  unsigned long long* corrections;
};

// Index of the largest E2M1 level (0, .5, 1, 1.5, 2, 3, 4, 6) at or below |v|,
// for both floats of a pair at once, in two 16-bit lanes: [level(lo) |
// level(hi) << 16].  The levels from 1 up are the floats 2^e (1 + m/2) with e
// in 0..2 and one mantissa bit m, so for |v| >= 1 the index is 2 + 2 e + m =
// f - 252 with f = exponent field * 2 + top mantissa bit (capped at 7);
// [0.5, 1) (f = 252, 253) is level 1 and anything below 0.5 (zeros,
// subnormals) level 0.  With f clamped to [251, 259] that is f - 251, less
// one for f >= 253.
__device__ __forceinline__ uint32_t floor_level2(uint64_t y) {
  const uint32_t w = __byte_perm(static_cast<uint32_t>(y), static_cast<uint32_t>(y >> 32), 0x7632);
  const uint32_t f = (w >> 6) & 0x01FF01FFu;      // the sign bits fall outside the mask
  uint32_t a;
  asm("max.u16x2 %0, %1, %2;" : "=r"(a) : "r"(f), "r"(0x00FB00FBu));
  asm("min.u16x2 %0, %0, %1;" : "+r"(a) : "r"(0x01030103u));
  const uint32_t ge = ((a + 0x00030003u) >> 8) & 0x00010001u;
  return a - 0x00FB00FBu - ge;
}

// Shared-memory group table (and, for few groups, the scale table tab);
// returns the number of rows that belong to a group.
__device__ __forceinline__ int64_t load_groups(const DirArgs& a, int32_t* off_s, float* g_s, float2* tab) {
  const int n = a.n_groups;
  for (int i = threadIdx.x; i <= n; i += blockDim.x) {
    off_s[i] = a.group_off ? a.group_off[i] : 0;
    if (i < n) g_s[i] = a.g[i];
  }
  if (n <= kDirTabGroups)
    for (int i = threadIdx.x; i < n * 128; i += blockDim.x) tab[i] = scale_table_entry(i & 127, a.g[i >> 7]);
  __syncthreads();
  return a.group_off ? min(a.rows, static_cast<int64_t>(off_s[n])) : a.rows;
}

__global__ void __launch_bounds__(kThreads, 4) direction_bits_kernel(DirArgs a) {
  extern __shared__ float2 smem_tab[];
  const bool use_tab = a.n_groups <= kDirTabGroups;
  float2* tab = smem_tab;                                          // n x 128 {S, 1/S} (few groups)
  int32_t* smem = reinterpret_cast<int32_t*>(smem_tab + (use_tab ? a.n_groups * 128 : 0));
  int32_t* off_s = smem;
  float* g_s = reinterpret_cast<float*>(smem + a.n_groups + 1);
  const int64_t rows = load_groups(a, off_s, g_s, tab);
  const RowGroups grp{a.group_off ? off_s : nullptr, a.n_groups, a.uniform};
  const int64_t K = a.K;
  const int nkb = static_cast<int>(K / 16);
  const int64_t ncol_tiles = ceil_div(nkb, 4);
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); row < rows;
       row += warps) {
    const int gi = grp.of(row);
    const float g = g_s[gi];
    const float2* tab_g = tab + gi * 128;
    for (int kb0 = lane; kb0 < nkb; kb0 += 64) {
      // both blocks' loads first: two 32-byte rows of x in flight per lane
      uint32_t w[2][8], sc[2];
      uint2 c[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int kb = kb0 + 32 * u;
        if (kb < nkb) {
          sc[u] = a.scales[a.tiled ? tiled_scale_offset(row, kb, ncol_tiles) : row * nkb + kb];
          load_bf16x16(a.x + row * K + kb * 16, w[u]);
          c[u] = __ldg(reinterpret_cast<const uint2*>(a.codes + row * (K / 2) + kb * 8));
        }
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int kb = kb0 + 32 * u;
        if (kb >= nkb) break;
        const float2 e = use_tab ? tab_g[sc[u] & 127u] : scale_table_entry(sc[u], g);
        uint32_t out = 0;
        if (e.x != 0.0f) {
          // level nibbles F of 8 elements per word, then per nibble
          // C > F  <=>  C + (7 - F) >= 8: bit 3 of C + (F ^ 7), no carry out
          // of a nibble (at most 14); bit 3 of nibble i moved to bit i
          const uint64_t inv2 = pack_f32x2(e.y, e.y);
          uint32_t f[2] = {0u, 0u};
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint32_t l2 = floor_level2(fmul2_rn(bf16x2_to_f32x2(w[u][i]), inv2));
            f[i >> 2] |= ((l2 | (l2 >> 12)) & 0xFFu) << (8 * (i & 3));
          }
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t cm = (h ? c[u].y : c[u].x) & 0x77777777u;
            uint32_t m = ((cm + (f[h] ^ 0x77777777u)) >> 3) & 0x11111111u;   // bit 4i = element i
            m = (m | (m >> 3)) & 0x03030303u;
            m = (m | (m >> 6)) & 0x000F000Fu;
            m = (m | (m >> 12)) & 0xFFu;
            out |= m << (8 * h);
          }
        }
        *reinterpret_cast<uint16_t*>(a.bits + row * (K / 8) + kb * 2) = static_cast<uint16_t>(out);
      }
    }
  }
}

__global__ void __launch_bounds__(kThreads, 3) replay_direction_kernel(DirArgs a) {
  extern __shared__ float2 smem_tab[];
  const int n = a.n_groups;
  const bool use_tab = n <= kDirTabGroups;
  float2* tab = smem_tab;                                          // n x 128 {S, 1/S} (few groups)
  int32_t* smem = reinterpret_cast<int32_t*>(smem_tab + (use_tab ? n * 128 : 0));
  const int64_t K = a.K;
  const int nkb = static_cast<int>(K / 16);
  const int npass = (nkb + 31) / 32;
  int32_t* off_s = smem;                                      // n + 1
  float* g_s = reinterpret_cast<float*>(smem + n + 1);        // n
  int32_t* pass_slot = smem + 2 * n + 1;                      // npass + 1
  int32_t* chan_s = pass_slot + npass + 1;                    // n_chan
  for (int j = threadIdx.x; j < a.n_chan; j += blockDim.x) chan_s[j] = a.chan[j];
  __syncthreads();
  for (int p = threadIdx.x; p <= npass && a.n_chan; p += blockDim.x) {
    int cnt = 0;                 // valid channels (ascending, first) below column 512 p
    for (int j = 0; j < a.n_chan; ++j) cnt += (chan_s[j] >= 0 && chan_s[j] < K && chan_s[j] < 512 * p) ? 1 : 0;
    pass_slot[p] = cnt;
  }
  const int64_t rows = load_groups(a, off_s, g_s, tab);
  const RowGroups grp{a.group_off ? off_s : nullptr, n, a.uniform};
  const int64_t ncol_tiles = ceil_div(nkb, 4);
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  uint32_t fixes = 0;
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); row < rows;
       row += warps) {
    const int gi = grp.of(row);
    const float g = g_s[gi];
    const float2* tab_g = tab + gi * 128;
    for (int p0 = 0; p0 < npass; p0 += 2) {
      // both passes' loads first: two 32-byte rows of x_train in flight per lane
      uint32_t wx[2][8], sx[2], bx[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int kb = (p0 + u) * 32 + lane;
        if (kb < nkb) {
          sx[u] = a.scales[a.tiled ? tiled_scale_offset(row, kb, ncol_tiles) : row * nkb + kb];
          bx[u] = *reinterpret_cast<const uint16_t*>(a.bits + row * (K / 8) + kb * 2);
          load_bf16x16(a.x + row * K + kb * 16, wx[u]);
        }
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int p = p0 + u;
        if (p >= npass) break;                              // warp-uniform
        const int kb = p * 32 + lane;
        QCore q{0u, 0u, 0u, 0.0f};
        if (kb < nkb) {
          const uint32_t s = sx[u];
          const float2 e = use_tab ? tab_g[s & 127u] : scale_table_entry(s, g);
          const uint32_t bits = bx[u];
          const uint32_t (&w)[8] = wx[u];
          q.scale = s;
          q.sv = e4m3_value(s);
          if (e.x == 0.0f) {
            // signed zeros, as the quantizer writes for a zero block scale
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              q.lo |= ((w[i] >> 15) & 1u) << (8 * i + 3) | ((w[i] >> 31) & 1u) << (8 * i + 7);
              q.hi |= ((w[4 + i] >> 15) & 1u) << (8 * i + 3) | ((w[4 + i] >> 31) & 1u) << (8 * i + 7);
            }
          } else {
            const uint64_t inv2 = pack_f32x2(e.y, e.y);
            uint64_t y[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) y[i] = fmul2_rn(bf16x2_to_f32x2(w[i]), inv2);
            // the trainer's own nearest-even codes carry y's sign (negative
            // zero included); the guided magnitudes are assembled nibble by
            // nibble, then the sign bits are taken from the own codes and the
            // differing magnitudes counted 8 at a time
            const uint32_t own_lo = e2m1x8_from_pairs(y), own_hi = e2m1x8_from_pairs(y + 4);
            uint32_t mag_lo = 0, mag_hi = 0;
            // bit 2i of the record to bit 0 and bit 2i + 1 to bit 16 of pair i
            const uint32_t spread = (bits & 0x5555u) | ((bits & 0xAAAAu) << 15);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              uint32_t l2 = floor_level2(y[i]) + ((spread >> (2 * i)) & 0x00010001u);
              asm("min.u16x2 %0, %0, %1;" : "+r"(l2) : "r"(0x00070007u));
              const uint32_t nib = (l2 | (l2 >> 12)) & 0xFFu;   // elements 2i and 2i + 1
              if (i < 4) mag_lo |= nib << (8 * i); else mag_hi |= nib << (8 * (i - 4));
            }
            q.lo = mag_lo | (own_lo & 0x88888888u);
            q.hi = mag_hi | (own_hi & 0x88888888u);
            uint32_t d0 = (mag_lo ^ own_lo) & 0x77777777u, d1 = (mag_hi ^ own_hi) & 0x77777777u;
            d0 = (d0 | (d0 >> 1) | (d0 >> 2)) & 0x11111111u;
            d1 = (d1 | (d1 >> 1) | (d1 >> 2)) & 0x11111111u;
            fixes += __popc(d0) + __popc(d1);
          }
          uint32_t o[8];
          deq_block_bf16(q, g, 1, o);
          uint4* dst = reinterpret_cast<uint4*>(a.x_hat + row * K + kb * 16);
          dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
          dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
          if (a.codes_out) *reinterpret_cast<uint2*>(a.codes_out + row * (K / 2) + kb * 8) = make_uint2(q.lo, q.hi);
        }
        if (a.n_chan)                // compensation channels of this pass: x_hat = bf16(fp32(deq) + r)
          replay_channel_pass(q, g, p, pass_slot[p], pass_slot[p + 1], chan_s, a.resid + row * a.n_chan,
                              a.x_hat + row * K);
      }
    }
  }
  if (a.corrections) {
    unsigned long long f = fixes;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) f += __shfl_xor_sync(0xffffffffu, f, o);
    if (lane == 0 && f) atomicAdd(a.corrections, f);
  }
}

int check_common(int64_t rows, int64_t K, const uint8_t* scales, int scale_layout, const float* g,
                 const int32_t* group_off, int n_groups) {
  QUADS_REQUIRE(rows >= 0 && K > 0 && K % 16 == 0 && K <= 65536, QUADS_ERR_UNSUPPORTED_SHAPE,
                "K must be a positive multiple of 16 up to 65536");
  QUADS_REQUIRE(rows * (K / 16) < (int64_t(1) << 31), QUADS_ERR_UNSUPPORTED_SHAPE, "tensor above 2^31 blocks");
  QUADS_REQUIRE(scale_layout == QUADS_SCALES_LINEAR || scale_layout == QUADS_SCALES_TILED, QUADS_ERR_INVALID_ARG,
                "unknown scale layout");
  QUADS_REQUIRE(n_groups >= 1 && n_groups <= kMaxGroups, QUADS_ERR_UNSUPPORTED_SHAPE, "n_groups must be in [1, %d]",
                kMaxGroups);
  QUADS_REQUIRE(group_off || rows % n_groups == 0, QUADS_ERR_INVALID_ARG,
                "without group offsets, rows must be a multiple of n_groups");
  QUADS_REQUIRE(rows == 0 || (scales && g), QUADS_ERR_INVALID_ARG, "scales and g must be non-null");
  return QUADS_OK;
}

DirArgs base_args(int64_t rows, int64_t K, const uint8_t* scales, int scale_layout, const float* g,
                  const int32_t* group_off, int n_groups) {
  DirArgs a{};
  a.scales = scales;
  a.tiled = scale_layout == QUADS_SCALES_TILED;
  a.g = g;
  a.group_off = group_off;
  a.n_groups = n_groups;
  a.uniform = make_fastdiv(static_cast<uint32_t>(n_groups > 1 && !group_off ? rows / n_groups : 1));
  a.rows = rows;
  a.K = K;
  return a;
}

}  // namespace
}  // namespace quads

using namespace quads;

extern "C" {

int trace_direction_bits(const uint16_t* x, int64_t rows, int64_t K, const uint8_t* codes, const uint8_t* scales,
                         int scale_layout, const float* g, const int32_t* group_off, int n_groups, uint8_t* bits,
                         quads_stream_t stream) {
  clear_error();
  QUADS_TRY(check_common(rows, K, scales, scale_layout, g, group_off, n_groups));
  if (rows == 0) return QUADS_OK;
  QUADS_REQUIRE(x && codes && bits && aligned(x, 16) && aligned(codes, 8) && aligned(bits, 2), QUADS_ERR_INVALID_ARG,
                "x (16-byte aligned), codes (8) and bits (2) must be non-null and aligned");
  DirArgs a = base_args(rows, K, scales, scale_layout, g, group_off, n_groups);
  a.x = x;
  a.codes = codes;
  a.bits = bits;
  const size_t smem = dir_tab_bytes(n_groups) + (2 * static_cast<size_t>(n_groups) + 1) * 4;
  const int grid = persistent_grid(reinterpret_cast<const void*>(direction_bits_kernel), kThreads, smem,
                                   ceil_div(rows, kThreads / 32));
  direction_bits_kernel<<<grid, kThreads, smem, stream>>>(a);
  count_launches(1);
  return check_launch("direction_bits_kernel");
}

int trace_replay_direction(const uint8_t* bits, const uint8_t* scales, int scale_layout, const float* g,
                           const int32_t* group_off, int n_groups, int64_t rows, int64_t K, const uint16_t* x_train,
                           const int32_t* chan, int n_chan, const uint16_t* resid, uint16_t* x_hat,
                           uint8_t* codes_out, unsigned long long* corrections, quads_stream_t stream) {
  clear_error();
  QUADS_TRY(check_common(rows, K, scales, scale_layout, g, group_off, n_groups));
  QUADS_REQUIRE(n_chan >= 0 && n_chan <= kMaxChan, QUADS_ERR_UNSUPPORTED_SHAPE, "n_chan must be in [0, %d]",
                kMaxChan);
  QUADS_REQUIRE(n_chan == 0 || (chan && resid), QUADS_ERR_INVALID_ARG, "chan and resid required with n_chan > 0");
  if (rows == 0) return QUADS_OK;
  QUADS_REQUIRE(bits && x_train && x_hat && aligned(bits, 2) && aligned(x_train, 16) && aligned(x_hat, 16) &&
                    (!codes_out || aligned(codes_out, 8)),
                QUADS_ERR_INVALID_ARG, "bits (2), x_train and x_hat (16), codes_out (8): non-null and aligned");
  DirArgs a = base_args(rows, K, scales, scale_layout, g, group_off, n_groups);
  a.x = x_train;
  a.bits = const_cast<uint8_t*>(bits);
  a.chan = chan;
  a.n_chan = n_chan;
  a.resid = resid;
  a.x_hat = x_hat;
  a.codes_out = codes_out;
  a.corrections = corrections;
  const size_t smem =
      dir_tab_bytes(n_groups) + (2 * static_cast<size_t>(n_groups) + 1 + (K / 16 + 31) / 32 + 1 + n_chan) * 4;
  if (smem > 48 * 1024 && cudaFuncSetAttribute(replay_direction_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(smem)) != cudaSuccess)
    return set_error(QUADS_ERR_CUDA, "cannot raise shared memory of replay_direction_kernel");
  const int grid = persistent_grid(reinterpret_cast<const void*>(replay_direction_kernel), kThreads, smem,
                                   ceil_div(rows, kThreads / 32));
  replay_direction_kernel<<<grid, kThreads, smem, stream>>>(a);
  count_launches(1);
  return check_launch("replay_direction_kernel");
}

}  // extern "C"
