// NVFP4 quantization kernels: per-group amax, quantize (+ residual channels,
// + weight fake-quant outputs), dequantize, channel calibration, STE backward.
//
// Method: [TRACE] "Fonctionnement, côté ingénierie" (block scaling, one 4-bit
// value per element, rounding direction as a discrete choice); [format]
// (16-element blocks along K, E4M3 block scale, FP32 per-tensor scale);
// [QUADS-fr §2.2.B] (residual on the high-residual channels);
// [QUADS-fr §2.2.A] (trainer weights fake-quantized onto the rollout's grid,
// straight-through backward).
//
// Every kernel is HBM-bound.  amax and quantize take one warp per row: a lane
// owns one 16-element block per pass (32 bytes of BF16 in; 8 bytes of codes
// and one scale byte out), a pass covers 32 consecutive blocks (1 KB), and a
// warp keeps two passes of loads in flight.  Grids are persistent: as many
// CTAs as fit on the SMs at once.  The elementwise kernels (dequantize, STE
// backward) are grid-stride loops.
#include <cstdio>
#include <mutex>

#include "common.cuh"

namespace quads {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxGroupsSmem = 1024;
constexpr int kMaxChan = 256;
constexpr int kTabGroups = 16;     // up to this many groups get a {S, 1/S} table in shared memory
constexpr int64_t kMaxBlocks = int64_t(1) << 31;

int grid_for(int64_t work, int per_block = kThreads) {
  int64_t g = ceil_div(work, per_block);
  int64_t cap = static_cast<int64_t>(num_sms()) * 16;
  if (g > cap) g = cap;
  if (g < 1) g = 1;
  return static_cast<int>(g);
}

// --------------------------------------------------------------------- amax

// One warp per row; each lane reads 32 bytes (16 elements) per pass, four
// passes in flight; |x| maxima on the BF16 bit patterns, two per word.
__global__ void __launch_bounds__(kThreads) amax_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t K,
                                                        int64_t ld, const int32_t* group_off, int n_groups,
                                                        FastDiv uniform, unsigned int* __restrict__ out_bits) {
  extern __shared__ int32_t smem[];
  int32_t* off_s = smem;                                   // n_groups + 1 (explicit groups)
  unsigned int* amax_s = reinterpret_cast<unsigned int*>(smem + n_groups + 1);
  for (int i = threadIdx.x; i <= n_groups; i += blockDim.x) {
    if (group_off != nullptr) off_s[i] = group_off[i];
    if (i < n_groups) amax_s[i] = 0u;
  }
  __syncthreads();
  RowGroups grp{group_off ? off_s : nullptr, n_groups, uniform};
  if (group_off != nullptr) rows = min(rows, static_cast<int64_t>(off_s[n_groups]));   // rows past the last group
  const int lane = threadIdx.x & 31;
  const int nkb = static_cast<int>(K / 16);
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  // each warp takes rows r and r + warps together: 4 loads of 32 bytes per lane in flight
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); row < rows;
       row += 2 * warps) {
    const int64_t row2 = row + warps;
    const bool two = row2 < rows;
    uint32_t m = 0u, m2 = 0u;
    for (int kb0 = 0; kb0 < nkb; kb0 += 2 * 32) {
      uint32_t w[4][8];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int kb = kb0 + (u & 1) * 32 + lane;
        const int64_t r = (u < 2) ? row : row2;
        if (kb < nkb && (u < 2 || two)) load_bf16x16(x + r * ld + kb * 16, w[u]);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int kb = kb0 + (u & 1) * 32 + lane;
        if (kb < nkb && (u < 2 || two)) {
          uint32_t& acc = (u < 2) ? m : m2;
#pragma unroll
          for (int i = 0; i < 8; ++i) acc = __vmaxu2(acc, w[u][i] & 0x7FFF7FFFu);
        }
      }
    }
    const unsigned int wm = __reduce_max_sync(0xffffffffu, max(m & 0xFFFFu, m >> 16));
    const unsigned int wm2 = __reduce_max_sync(0xffffffffu, max(m2 & 0xFFFFu, m2 >> 16));
    if (lane == 0) {
      if (wm) atomicMax(&amax_s[grp.of(row)], wm);
      if (two && wm2) atomicMax(&amax_s[grp.of(row2)], wm2);
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < n_groups; i += blockDim.x)
    if (amax_s[i]) atomicMax(&out_bits[i], amax_s[i] << 16);
}

// Contiguous rows (ld == K): one sweep over the tensor in warp chunks of
// 256 16-byte vectors (4 KB, lane l loads vectors l, l + 32, ... of the chunk:
// eight coalesced 512-byte loads in flight per warp), chunks grid-strided
// over the warps.  Groups are long contiguous ranges, so a chunk almost
// always lies in one group, found once per chunk; a thread keeps a running
// maximum for its current group and folds it into the block's shared maxima
// when the group changes; the block then folds those into the output.
constexpr int kAmaxUnroll = 8;
constexpr uint32_t kAmaxChunk = 32 * kAmaxUnroll;

__global__ void __launch_bounds__(kThreads) amax_flat_kernel(const uint4* __restrict__ x, int64_t rows,
                                                             uint32_t vec_per_row, const int32_t* group_off,
                                                             int n_groups, FastDiv vec_div, FastDiv uniform,
                                                             unsigned int* __restrict__ out_bits) {
  extern __shared__ int32_t sm_a[];
  int32_t* off_a = sm_a;                                   // n_groups + 1 (explicit groups)
  unsigned int* am_a = reinterpret_cast<unsigned int*>(sm_a + n_groups + 1);
  for (int i = threadIdx.x; i <= n_groups; i += blockDim.x) {
    if (group_off != nullptr) off_a[i] = group_off[i];
    if (i < n_groups) am_a[i] = 0u;
  }
  __syncthreads();
  RowGroups grp{group_off ? off_a : nullptr, n_groups, uniform};
  if (group_off != nullptr) rows = min(rows, static_cast<int64_t>(off_a[n_groups]));   // rows past the last group
  const uint32_t nvec = static_cast<uint32_t>(rows * vec_per_row);   // < 2^31 (checked on the host)
  const uint32_t lane = threadIdx.x & 31;
  const uint32_t nwarps = gridDim.x * (blockDim.x >> 5);
  const uint32_t nchunks = (nvec + kAmaxChunk - 1) / kAmaxChunk;
  int cur = -1;
  uint32_t m = 0u;
  auto fold = [&](int g) {
    const unsigned int mm = max(m & 0xFFFFu, m >> 16);
    if (cur >= 0 && mm) atomicMax(&am_a[cur], mm);
    cur = g;
    m = 0u;
  };
  for (uint32_t c = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); c < nchunks; c += nwarps) {
    const uint32_t base = c * kAmaxChunk;
    uint4 r[kAmaxUnroll];
#pragma unroll
    for (int u = 0; u < kAmaxUnroll; ++u) {
      const uint32_t v = base + u * 32 + lane;
      r[u] = v < nvec ? __ldg(x + v) : make_uint4(0u, 0u, 0u, 0u);
    }
    const uint32_t last = min(base + kAmaxChunk, nvec) - 1;
    const int g0 = grp.of(fast_div(base, vec_div));
    const bool one_group = g0 == grp.of(fast_div(last, vec_div));
#pragma unroll
    for (int u = 0; u < kAmaxUnroll; ++u) {
      const uint32_t v = base + u * 32 + lane;
      if (v >= nvec) break;
      const int g = one_group ? g0 : grp.of(fast_div(v, vec_div));
      if (g != cur) fold(g);
      m = __vmaxu2(m, r[u].x & 0x7FFF7FFFu);
      m = __vmaxu2(m, r[u].y & 0x7FFF7FFFu);
      m = __vmaxu2(m, r[u].z & 0x7FFF7FFFu);
      m = __vmaxu2(m, r[u].w & 0x7FFF7FFFu);
    }
  }
  fold(-1);
  __syncthreads();
  for (int i = threadIdx.x; i < n_groups; i += blockDim.x)
    if (am_a[i]) atomicMax(&out_bits[i], am_a[i] << 16);
}

// ----------------------------------------------------------------- quantize

struct QuantArgs {
  const uint16_t* x;
  int64_t rows, K, ld;
  const int32_t* group_off;
  int n_groups;
  int64_t uniform_rows;
  const float* amax;       // [n_groups]
  uint8_t* codes;          // [rows][K/2] or null
  uint8_t* scales;         // or null
  int scale_layout;
  float* g_out;            // [n_groups] or null
  const int32_t* chan;     // [n_chan]
  int n_chan;
  uint16_t* resid;         // [rows][n_chan] or null
  int resid_mode;          // 0: residual, 1: bf16(deq), 2: the input itself
  uint16_t* w_fq;          // [rows][K] or null
  int fold;                // w_fq = bf16(deq) (1) or e2m1 * e4m3 (0)
  int64_t ilv_half;        // > 0: codes, scales and resid rows of each group of
                           // 2 * ilv_half rows interleaved in blocks of 64 (first
                           // half 64 rows, second half 64 rows, ...); 0: input order
  FastDiv uniform_div;     // filled by launch_quantize: rows per group (uniform groups)
};

// One warp per row, lanes along K (32 blocks of 16 elements per pass, two
// passes in flight).  The residual channels of a pass are extracted
// cooperatively: lane j takes channel slot j and fetches its element, code and
// scale from the lane that owns the block by warp shuffles, then the warp
// writes the row's residual slots as one contiguous store.
// kMode: 0 any combination of outputs (runtime checks); 1 the weight
// fake-quant (codes, scales, W_fq with g folded, compensation columns as
// bf16(deq)); 2 the activation quantizer (codes, scales, residual channels).
// Eight words to 32-byte aligned shared memory.
__device__ __forceinline__ void st_shared_u32x8(uint32_t* p, const uint32_t (&o)[8]) {
  reinterpret_cast<uint4*>(p)[0] = make_uint4(o[0], o[1], o[2], o[3]);
  reinterpret_cast<uint4*>(p)[1] = make_uint4(o[4], o[5], o[6], o[7]);
}

template <int kMode>
__global__ void __launch_bounds__(kThreads, 4) quantize_kernel(QuantArgs a) {
  constexpr bool kFq = kMode == 1, kAct = kMode == 2;
  // passes of a row whose 32-byte loads are in flight at once (the
  // activation quantizer's per-block work is lighter: more loads cover it)
  constexpr int kU = kAct ? 4 : 2;
  const bool has_codes = kFq || kAct || a.codes != nullptr;
  const bool has_scales = kFq || kAct || a.scales != nullptr;
  const bool has_wfq = kFq || (!kAct && a.w_fq != nullptr);
  const int fold = kFq ? 1 : a.fold;
  const int resid_mode = kFq ? 1 : (kAct ? 0 : a.resid_mode);
  extern __shared__ int32_t smem_q[];
  // weight fake-quant: each warp's W_fq words of the current pass (32 lanes x
  // 8 words), from which the compensation columns are picked
  __shared__ __align__(16) uint32_t wfq_s[kFq ? (kThreads / 32) * 32 * 8 : 4];
  // residual channels of the other modes: each warp's inputs (32 lanes x 8
  // words), codes (32 x 2 words) and block scale values (32 words) of the
  // current pass, from which the channel slots pick their element
  constexpr int kXqWords = 32 * 8 + 32 * 2 + 32;
  __shared__ __align__(16) uint32_t xq_s[kFq ? 4 : (kThreads / 32) * kXqWords];
  const int n = a.n_groups;
  const int nkb = static_cast<int>(a.K / 16);
  const int npass = (nkb + 31) / 32;
  const bool use_tab = n <= kTabGroups;
  float2* tab = reinterpret_cast<float2*>(smem_q);         // n x 128 {S, 1/S} (few groups)
  int32_t* smem = smem_q + (use_tab ? n * 128 * 2 : 0);
  int32_t* off_s = smem;                                   // n + 1
  float* g_s = reinterpret_cast<float*>(smem + n + 1);     // n
  int32_t* pass_slot = smem + 2 * n + 1;                   // npass + 1 (with channels)
  int32_t* chan_s = pass_slot + npass + 1;                 // n_chan
  __shared__ int n_valid_s;
  for (int i = threadIdx.x; i <= n; i += blockDim.x) {
    if (a.group_off != nullptr) off_s[i] = a.group_off[i];
    if (i < n) {
      const float g = __fdiv_rn(a.amax[i], kNvfp4Range);
      g_s[i] = g;
      if (blockIdx.x == 0 && a.g_out != nullptr) a.g_out[i] = g;
    }
  }
  if (use_tab)
    for (int i = threadIdx.x; i < n * 128; i += blockDim.x)
      tab[i] = scale_table_entry(i & 127, __fdiv_rn(a.amax[i >> 7], kNvfp4Range));
  if (a.n_chan) {
    for (int j = threadIdx.x; j < a.n_chan; j += blockDim.x) chan_s[j] = a.chan[j];
    __syncthreads();
    // valid channels are ascending and first: slots of pass p are
    // [#valid < 512 p, #valid < 512 (p + 1))
    for (int p = threadIdx.x; p <= npass; p += blockDim.x) {
      int cnt = 0;
      for (int j = 0; j < a.n_chan; ++j) {
        const int c = chan_s[j];
        cnt += (c >= 0 && c < a.K && c < 512 * p) ? 1 : 0;
      }
      pass_slot[p] = cnt;
    }
    if (threadIdx.x == 0) {
      int cnt = 0;
      for (int j = 0; j < a.n_chan; ++j) cnt += (chan_s[j] >= 0 && chan_s[j] < a.K) ? 1 : 0;
      n_valid_s = cnt;
    }
  }
  __syncthreads();
  RowGroups grp{a.group_off ? off_s : nullptr, n, a.uniform_div};
  const bool tiled = a.scale_layout == QUADS_SCALES_TILED;
  const int64_t rows_valid = a.group_off ? min(a.rows, static_cast<int64_t>(off_s[n])) : a.rows;
  const int64_t rows_e = tiled ? ceil_div(rows_valid, 128) * 128 : rows_valid;
  const int nkb_e = tiled ? (nkb + 3) / 4 * 4 : nkb;
  const int64_t ncol_tiles = nkb_e / 4;
  const int n_valid = a.n_chan ? n_valid_s : 0;
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); row < rows_e;
       row += warps) {
    if (row >= rows_valid) {                           // padding rows of the last tiled band
      if (has_scales)
        for (int kb = lane; kb < nkb_e; kb += 32) a.scales[tiled_scale_offset(row, kb, ncol_tiles)] = 0;
      continue;
    }
    const int gi = grp.of(row);
    const float g = g_s[gi];
    const QConsts qc = make_qconsts(g, use_tab ? tab + gi * 128 : nullptr);
    const uint16_t* xr = a.x + row * a.ld;
    int64_t drow = row;                                // row of the codes, scales and resid outputs
    if (a.ilv_half) {
      const int64_t base = static_cast<int64_t>(gi) * 2 * a.ilv_half, loc = row - base;
      const bool second = loc >= a.ilv_half;
      const int64_t f = second ? loc - a.ilv_half : loc;
      drow = base + (f >> 6) * 128 + (second ? 64 : 0) + (f & 63);
    }
    // the row's part of the scale offsets (tiled: band, lane and quarter of the row)
    const int64_t sbase = tiled ? ((drow >> 7) * ncol_tiles) * 512 + (drow & 31) * 16 + ((drow >> 5) & 3) * 4
                                : drow * nkb;
    for (int p0 = 0; p0 < npass; p0 += kU) {
      uint32_t w[kU][8];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int kb = (p0 + u) * 32 + lane;
        if (kb < nkb) load_bf16x16(xr + kb * 16, w[u]);
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int p = p0 + u;
        if (p >= npass) break;                         // warp-uniform
        const int kb = p * 32 + lane;
        QCore q{0u, 0u, 0u, 0.0f};
        uint32_t o[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
        if (kb < nkb) {
          q = quant_core(w[u], qc);
          if (has_codes)
            *reinterpret_cast<uint2*>(a.codes + drow * (a.K / 2) + kb * 8) = make_uint2(q.lo, q.hi);
          if (has_wfq) {
            deq_block_bf16(q, g, fold, o);
            uint4* dst = reinterpret_cast<uint4*>(a.w_fq + row * a.K + kb * 16);
            dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
            dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
          }
        }
        if (has_scales && kb < nkb_e)
          a.scales[sbase + (tiled ? (kb >> 2) * 512 + (kb & 3) : kb)] = static_cast<uint8_t>(q.scale);
        if (kFq && a.resid) {
          // The compensation column of channel c is W_fq[:, c] itself (the
          // fold makes bf16(deq) the W_fq value): the warp stages its W_fq
          // words of the pass and channel slot j takes lane j % 32, which
          // picks its element there.
          const int slo = pass_slot[p], shi = pass_slot[p + 1];
          if (slo < shi) {                                 // warp-uniform
            uint32_t* const ws = wfq_s + (threadIdx.x >> 5) * 256;
            st_shared_u32x8(ws + lane * 8, o);
            __syncwarp();
            for (int j0 = slo; j0 < shi; j0 += 32) {
              const int j = j0 + lane;
              if (j < shi) {
                const int c = chan_s[j] - 512 * p;
                const uint32_t word = ws[(c >> 4) * 8 + ((c & 15) >> 1)];
                a.resid[drow * a.n_chan + j] = static_cast<uint16_t>((c & 1) ? (word >> 16) : (word & 0xFFFFu));
              }
            }
            __syncwarp();
          }
        } else if (a.resid) {
          // Channel slot j of this pass is taken by lane j % 32, which picks
          // the element's input, code and block scale from the warp's staged
          // pass.  bf16(deq) = bf16(fp32(val(q) val(s)) g) is the W_fq value.
          const int slo = pass_slot[p], shi = pass_slot[p + 1];
          if (slo < shi) {                                 // warp-uniform
            uint32_t* const xs = xq_s + (threadIdx.x >> 5) * kXqWords;
            st_shared_u32x8(xs + lane * 8, w[u]);
            xs[256 + 2 * lane] = q.lo;
            xs[257 + 2 * lane] = q.hi;
            xs[320 + lane] = __float_as_uint(q.sv);
            __syncwarp();
            for (int j0 = slo; j0 < shi; j0 += 32) {
              const int j = j0 + lane;
              if (j < shi) {
                const int c = chan_s[j] - 512 * p;         // column within the pass
                const int src = c >> 4, bit = c & 15;
                const uint32_t code = (xs[256 + 2 * src + (bit >> 3)] >> (4 * (bit & 7))) & 15u;
                const float sv = __uint_as_float(xs[320 + src]);
                float v;
                if (resid_mode == 1) {
                  v = deq_f32(code, sv, g);
                } else {
                  const uint32_t xw = xs[8 * src + (bit >> 1)];
                  const float xv = bf16_bits_to_float((bit & 1) ? (xw >> 16) : (xw & 0xFFFFu));
                  v = (resid_mode == 2) ? xv : __fsub_rn(xv, deq_f32(code, sv, g));
                }
                a.resid[drow * a.n_chan + j] = static_cast<uint16_t>(float_to_bf16_bits(v));
              }
            }
            __syncwarp();
          }
        }
      }
    }
    if (a.resid)
      for (int j = n_valid + lane; j < a.n_chan; j += 32) a.resid[drow * a.n_chan + j] = 0;
  }
}

size_t quantize_smem(int n_groups, int64_t K, int n_chan) {
  size_t s = (2 * static_cast<size_t>(n_groups) + 1) * 4;
  if (n_groups <= kTabGroups) s += static_cast<size_t>(n_groups) * 128 * sizeof(float2);
  if (n_chan) s += (static_cast<size_t>((K / 16 + 31) / 32) + 1 + n_chan) * 4;
  return s;
}

// --------------------------------------------------------------- dequantize

__global__ void __launch_bounds__(kThreads) dequant_kernel(const uint8_t* __restrict__ codes,
                                                           const uint8_t* __restrict__ scales, int layout,
                                                           const float* __restrict__ g, const int32_t* group_off,
                                                           int n_groups, FastDiv uniform, uint32_t total,
                                                           uint32_t nkb, FastDiv nkb_div, int64_t K, void* out,
                                                           int out_dtype) {
  extern __shared__ int32_t smem[];
  for (int i = threadIdx.x; i <= n_groups; i += blockDim.x)
    if (group_off) smem[i] = group_off[i];
  __syncthreads();
  RowGroups grp{group_off ? smem : nullptr, n_groups, uniform};
  const uint32_t ncol_tiles = (nkb + 3) / 4;
  const uint32_t stride = gridDim.x * blockDim.x;
  for (uint32_t b = blockIdx.x * blockDim.x + threadIdx.x; b < total; b += stride) {
    const uint32_t row = fast_div(b, nkb_div), kb = b - row * nkb;
    const uint2 c = __ldg(reinterpret_cast<const uint2*>(codes + static_cast<int64_t>(row) * (K / 2) + kb * 8));
    const uint32_t s = scales[layout == QUADS_SCALES_TILED ? tiled_scale_offset(row, kb, ncol_tiles)
                                                           : static_cast<int64_t>(b)];
    const float sv = e4m3_value(s);
    const float gg = g[grp.of(row)];
    float v[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      v[i] = deq_f32((c.x >> (4 * i)) & 15u, sv, gg);
      v[8 + i] = deq_f32((c.y >> (4 * i)) & 15u, sv, gg);
    }
    if (out_dtype == QUADS_OUT_F32) {
      float4* d = reinterpret_cast<float4*>(static_cast<float*>(out) + static_cast<int64_t>(row) * K + kb * 16);
#pragma unroll
      for (int i = 0; i < 4; ++i) d[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    } else {
      uint4* d = reinterpret_cast<uint4*>(static_cast<uint16_t*>(out) + static_cast<int64_t>(row) * K + kb * 16);
      d[0] = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                        pack_bf16x2(v[6], v[7]));
      d[1] = make_uint4(pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]), pack_bf16x2(v[12], v[13]),
                        pack_bf16x2(v[14], v[15]));
    }
  }
}

// ------------------------------------------------------ channel calibration

constexpr int kScoreRows = 256;   // rows per partial sum

// partial[chunk][K]: sum over the chunk's rows (in row order) of |fp32 residual|.
__global__ void __launch_bounds__(kThreads) channel_partial_kernel(const uint16_t* __restrict__ x,
                                                                   int64_t rows, int64_t K,
                                                                   const float* __restrict__ amax,
                                                                   float* __restrict__ partial) {
  const int64_t nkb = K / 16;
  const int64_t kb = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t chunk = blockIdx.y;
  if (kb >= nkb) return;
  const float g = __fdiv_rn(amax[0], kNvfp4Range);
  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.0f;
  const int64_t r0 = chunk * kScoreRows, r1 = min(rows, r0 + kScoreRows);
  for (int64_t row = r0; row < r1; ++row) {
    QBlock q;
    uint32_t w[8];
    load_bf16x16(x + row * K + kb * 16, w);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      q.x[2 * i] = bf16_bits_to_float(w[i] & 0xFFFFu);
      q.x[2 * i + 1] = bf16_bits_to_float(w[i] >> 16);
    }
    quantize_block(q, g);
#pragma unroll
    for (int i = 0; i < 16; ++i)
      acc[i] = __fadd_rn(acc[i], fabsf(__fsub_rn(q.x[i], deq_f32(qblock_code(q, i), q.sv, g))));
  }
  float* dst = partial + chunk * K + kb * 16;
#pragma unroll
  for (int i = 0; i < 16; ++i) dst[i] = acc[i];
}

__global__ void channel_reduce_kernel(const float* __restrict__ partial, int64_t n_chunks, int64_t K,
                                      float* __restrict__ scores) {
  int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (c >= K) return;
  float s = 0.0f;
  for (int64_t i = 0; i < n_chunks; ++i) s = __fadd_rn(s, partial[i * K + c]);
  scores[c] = s;
}

// One block: rank every channel by (score desc, index asc), keep rank < n_sel,
// write the kept channels in ascending order.
__global__ void __launch_bounds__(1024) select_kernel(const float* __restrict__ scores, int K, int n_sel,
                                                      int32_t* __restrict__ chan_out) {
  extern __shared__ float s_scores[];
  __shared__ int warp_tot[32];
  __shared__ int carry;
  for (int i = threadIdx.x; i < K; i += blockDim.x) s_scores[i] = scores[i];
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  for (int base = 0; base < K; base += blockDim.x) {
    int c = base + threadIdx.x;
    int keep = 0;
    if (c < K) {
      float v = s_scores[c];
      int rank = 0;
      for (int j = 0; j < K; ++j) {
        float u = s_scores[j];
        rank += (u > v) || (u == v && j < c);
      }
      keep = rank < n_sel;
    }
    unsigned int bal = __ballot_sync(0xffffffffu, keep);
    int before = __popc(bal & ((1u << lane) - 1u));
    if (lane == 0) warp_tot[wid] = __popc(bal);
    __syncthreads();
    int wbase = 0;
    for (int w = 0; w < wid; ++w) wbase += warp_tot[w];
    if (keep) chan_out[carry + wbase + before] = c;
    __syncthreads();
    if (threadIdx.x == 0) {
      int t = 0;
      for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += warp_tot[w];
      carry += t;
    }
    __syncthreads();
  }
}

// ------------------------------------------------------------ STE backward


// ------------------------------------------------------------- host helpers

int validate_matrix(const void* x, int64_t rows, int64_t K, int64_t ld) {
  QUADS_REQUIRE(rows >= 0 && K > 0, QUADS_ERR_INVALID_ARG, "rows must be >= 0 and K > 0");
  QUADS_REQUIRE(K % 16 == 0, QUADS_ERR_UNSUPPORTED_SHAPE, "K (%lld) must be a multiple of 16", (long long)K);
  QUADS_REQUIRE(K <= 65536, QUADS_ERR_UNSUPPORTED_SHAPE, "K (%lld) above 65536", (long long)K);
  QUADS_REQUIRE(ld >= K && ld % 8 == 0, QUADS_ERR_INVALID_ARG, "ld (%lld) must be >= K and a multiple of 8",
                (long long)ld);
  QUADS_REQUIRE(rows == 0 || (x != nullptr && aligned(x, 16)), QUADS_ERR_INVALID_ARG,
                "input must be non-null and 16-byte aligned");
  return QUADS_OK;
}

int validate_groups(const int32_t* group_off, int n_groups, int64_t rows) {
  QUADS_REQUIRE(n_groups >= 1, QUADS_ERR_INVALID_ARG, "n_groups must be >= 1");
  if (group_off) {
    QUADS_REQUIRE(n_groups <= kMaxGroupsSmem, QUADS_ERR_UNSUPPORTED_SHAPE, "n_groups above %d", kMaxGroupsSmem);
  } else {
    QUADS_REQUIRE(rows % n_groups == 0, QUADS_ERR_INVALID_ARG,
                  "without group offsets, rows (%lld) must be a multiple of n_groups (%d)", (long long)rows,
                  n_groups);
    QUADS_REQUIRE(n_groups <= kMaxGroupsSmem, QUADS_ERR_UNSUPPORTED_SHAPE, "n_groups above %d", kMaxGroupsSmem);
  }
  return QUADS_OK;
}

int launch_amax(const uint16_t* x, int64_t rows, int64_t K, int64_t ld, const int32_t* group_off, int n_groups,
                float* amax_out, cudaStream_t s) {
  if (cudaMemsetAsync(amax_out, 0, sizeof(float) * n_groups, s) != cudaSuccess)
    return set_error(QUADS_ERR_CUDA, "memset of the amax output failed");
  if (rows == 0) return QUADS_OK;
  QUADS_REQUIRE(rows < kMaxBlocks, QUADS_ERR_UNSUPPORTED_SHAPE, "too many rows");
  const uint32_t uniform = group_off ? 1u : static_cast<uint32_t>(rows / n_groups);
  if (ld == K && rows * (K / 8) < (int64_t(1) << 31)) {
    const size_t smem_f = (2 * static_cast<size_t>(n_groups) + 1) * 4;
    const int64_t nvec = rows * (K / 8);
    // four CTAs of 8 warps per SM: 128 KB per SM in flight
    const int64_t want = ceil_div(nvec, static_cast<int64_t>(kThreads) * kAmaxUnroll);
    const int grid_f = static_cast<int>(want < 4 * num_sms() ? (want < 1 ? 1 : want) : 4 * num_sms());
    amax_flat_kernel<<<grid_f, kThreads, smem_f, s>>>(reinterpret_cast<const uint4*>(x), rows,
                                                      static_cast<uint32_t>(K / 8), group_off, n_groups,
                                                      make_fastdiv(static_cast<uint32_t>(K / 8)),
                                                      make_fastdiv(uniform ? uniform : 1u),
                                                      reinterpret_cast<unsigned int*>(amax_out));
    count_launches(1);
    return check_launch("amax_flat_kernel");
  }
  size_t smem = (2 * static_cast<size_t>(n_groups) + 1) * 4;
  const int grid = persistent_grid(reinterpret_cast<const void*>(amax_kernel), kThreads, smem, ceil_div(rows, 16));
  amax_kernel<<<grid, kThreads, smem, s>>>(x, rows, K, ld, group_off, n_groups,
                                                          make_fastdiv(uniform ? uniform : 1u),
                                                          reinterpret_cast<unsigned int*>(amax_out));
  count_launches(1);
  return check_launch("amax_kernel");
}

template <int kMode>
int launch_quantize_mode(const QuantArgs& a, size_t smem, int64_t rows_e, cudaStream_t s) {
  if (smem > 48 * 1024 && cudaFuncSetAttribute(quantize_kernel<kMode>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(smem)) != cudaSuccess)
    return set_error(QUADS_ERR_CUDA, "cannot raise shared memory of quantize_kernel");
  const int grid = persistent_grid(reinterpret_cast<const void*>(quantize_kernel<kMode>), kThreads, smem,
                                   ceil_div(rows_e, 8));
  quantize_kernel<kMode><<<grid, kThreads, smem, s>>>(a);
  count_launches(1);
  return check_launch("quantize_kernel");
}

// Narrow rows (K <= 256) with codes and scales only: one thread per 16-element
// block instead of one warp per row, so that a row of a few blocks does not
// leave most lanes idle (the NVFP4 operands of the channel columns and
// residuals are 64 to 256 wide).  Same operations as quantize_kernel.
__global__ void __launch_bounds__(kThreads) quantize_narrow_kernel(QuantArgs a, FastDiv nkb_e_div) {
  extern __shared__ int32_t smem_n[];
  const int n = a.n_groups;
  int32_t* off_s = smem_n;                                   // n + 1
  float* g_s = reinterpret_cast<float*>(smem_n + n + 1);     // n
  for (int i = threadIdx.x; i <= n; i += blockDim.x) {
    if (a.group_off != nullptr) off_s[i] = a.group_off[i];
    if (i < n) {
      const float g = __fdiv_rn(a.amax[i], kNvfp4Range);
      g_s[i] = g;
      if (blockIdx.x == 0 && a.g_out != nullptr) a.g_out[i] = g;
    }
  }
  __syncthreads();
  const RowGroups grp{a.group_off ? off_s : nullptr, n, a.uniform_div};
  const bool tiled = a.scale_layout == QUADS_SCALES_TILED;
  const int nkb = static_cast<int>(a.K / 16);
  const int64_t rows_valid = a.group_off ? min(a.rows, static_cast<int64_t>(off_s[n])) : a.rows;
  const int64_t rows_e = tiled ? ceil_div(rows_valid, 128) * 128 : rows_valid;
  const int nkb_e = static_cast<int>(nkb_e_div.d);
  const int64_t ncol_tiles = nkb_e / 4;
  const uint32_t total = static_cast<uint32_t>(rows_e * nkb_e);
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += gridDim.x * blockDim.x) {
    const int64_t row = fast_div(i, nkb_e_div);
    const int kb = static_cast<int>(i - static_cast<uint32_t>(row) * nkb_e);
    const int64_t so = tiled ? tiled_scale_offset(row, kb, ncol_tiles) : row * nkb + kb;
    if (row >= rows_valid || kb >= nkb) {            // padding of the tiled layout
      a.scales[so] = 0;
      continue;
    }
    uint32_t w[8];
    load_bf16x16(a.x + row * a.ld + kb * 16, w);
    const QCore q = quant_core(w, g_s[grp.of(row)]);
    *reinterpret_cast<uint2*>(a.codes + row * (a.K / 2) + kb * 8) = make_uint2(q.lo, q.hi);
    a.scales[so] = static_cast<uint8_t>(q.scale);
  }
}

int launch_quantize(QuantArgs a, cudaStream_t s) {
  if (a.rows == 0) return QUADS_OK;
  QUADS_REQUIRE(a.rows < kMaxBlocks, QUADS_ERR_UNSUPPORTED_SHAPE, "too many rows");
  a.uniform_div = make_fastdiv(a.group_off ? 1u : static_cast<uint32_t>(a.uniform_rows > 0 ? a.uniform_rows : 1));
  const size_t smem = quantize_smem(a.n_groups, a.K, a.n_chan);
  const int64_t rows_e = a.scale_layout == QUADS_SCALES_TILED ? ceil_div(a.rows, 128) * 128 : a.rows;
  const bool any_resid = a.resid != nullptr && a.n_chan > 0;
  const int nkb = static_cast<int>(a.K / 16);
  const int nkb_e = a.scale_layout == QUADS_SCALES_TILED ? (nkb + 3) / 4 * 4 : nkb;
  if (a.codes && a.scales && !a.w_fq && !any_resid && a.ilv_half == 0 && nkb <= 16 &&
      rows_e * nkb_e < (int64_t(1) << 31)) {
    const size_t smem_n = (2 * static_cast<size_t>(a.n_groups) + 1) * 4;
    const int64_t blocks = ceil_div(rows_e * nkb_e, kThreads);
    const int64_t cap = static_cast<int64_t>(num_sms()) * 8;
    const int grid = static_cast<int>(blocks < cap ? blocks : cap);
    quantize_narrow_kernel<<<grid, kThreads, smem_n, s>>>(a, make_fastdiv(static_cast<uint32_t>(nkb_e)));
    count_launches(1);
    return check_launch("quantize_narrow_kernel");
  }
  if (a.codes && a.scales && a.w_fq && a.fold && (!any_resid || a.resid_mode == 1))
    return launch_quantize_mode<1>(a, smem, rows_e, s);
  if (a.codes && a.scales && !a.w_fq && (!any_resid || a.resid_mode == 0))
    return launch_quantize_mode<2>(a, smem, rows_e, s);
  return launch_quantize_mode<0>(a, smem, rows_e, s);
}

}  // namespace
}  // namespace quads

using namespace quads;

extern "C" {

size_t quads_quantize_workspace_bytes(int n_groups) {
  if (n_groups < 1) return 0;
  return static_cast<size_t>(ceil_div(static_cast<int64_t>(n_groups) * 4, 256) * 256);
}

int quads_amax_bf16(const uint16_t* x, int64_t rows, int64_t K, int64_t ld_x, const int32_t* group_off,
                    int n_groups, float* amax_out, quads_stream_t stream) {
  clear_error();
  QUADS_TRY(validate_matrix(x, rows, K, ld_x));
  QUADS_TRY(validate_groups(group_off, n_groups, rows));
  QUADS_REQUIRE(amax_out != nullptr, QUADS_ERR_INVALID_ARG, "amax_out is null");
  return launch_amax(x, rows, K, ld_x, group_off, n_groups, amax_out, stream);
}

int quads_quantize_nvfp4(const uint16_t* x, int64_t rows, int64_t K, int64_t ld_x, const int32_t* group_off,
                         int n_groups, const float* amax_in, uint8_t* codes, uint8_t* scales, int scale_layout,
                         float* g_out, const int32_t* chan, int n_chan, uint16_t* resid_out, void* ws,
                         size_t ws_bytes, quads_stream_t stream) {
  clear_error();
  QUADS_TRY(validate_matrix(x, rows, K, ld_x));
  QUADS_TRY(validate_groups(group_off, n_groups, rows));
  QUADS_REQUIRE(scale_layout == QUADS_SCALES_LINEAR || scale_layout == QUADS_SCALES_TILED,
                QUADS_ERR_INVALID_ARG, "unknown scale layout %d", scale_layout);
  QUADS_REQUIRE(g_out && (rows == 0 || (codes && scales)), QUADS_ERR_INVALID_ARG,
                "codes, scales and g_out must be non-null (codes and scales may be null for zero rows)");
  QUADS_REQUIRE(aligned(codes, 8), QUADS_ERR_INVALID_ARG, "codes must be 8-byte aligned");
  QUADS_REQUIRE(n_chan >= 0 && n_chan <= kMaxChan, QUADS_ERR_UNSUPPORTED_SHAPE, "n_chan must be in [0, %d]",
                kMaxChan);
  QUADS_REQUIRE(n_chan == 0 || (chan && resid_out), QUADS_ERR_INVALID_ARG,
                "chan and resid_out are required when n_chan > 0");
  const float* amax = amax_in;
  if (amax == nullptr) {
    QUADS_REQUIRE(ws != nullptr && ws_bytes >= quads_quantize_workspace_bytes(n_groups), QUADS_ERR_INVALID_ARG,
                  "workspace of %zu bytes required when amax_in is NULL", quads_quantize_workspace_bytes(n_groups));
    QUADS_TRY(launch_amax(x, rows, K, ld_x, group_off, n_groups, static_cast<float*>(ws), stream));
    amax = static_cast<const float*>(ws);
  }
  QuantArgs a{};
  a.x = x; a.rows = rows; a.K = K; a.ld = ld_x;
  a.group_off = group_off; a.n_groups = n_groups; a.uniform_rows = group_off ? 1 : (rows ? rows / n_groups : 1);
  a.amax = amax; a.codes = codes; a.scales = scales; a.scale_layout = scale_layout; a.g_out = g_out;
  a.chan = chan; a.n_chan = n_chan; a.resid = n_chan ? resid_out : nullptr; a.resid_mode = 0;
  a.w_fq = nullptr; a.fold = 1;
  if (rows == 0) {
    // still publish g (computed from the given or zero amax) and the padded scale tiles
    if (cudaMemsetAsync(g_out, 0, sizeof(float) * n_groups, stream) != cudaSuccess)
      return set_error(QUADS_ERR_CUDA, "memset failed");
    return QUADS_OK;
  }
  return launch_quantize(a, stream);
}

int quads_dequant(const uint8_t* codes, const uint8_t* scales, int scale_layout, const float* g,
                  const int32_t* group_off, int n_groups, int64_t rows, int64_t K, void* out, int out_dtype,
                  quads_stream_t stream) {
  clear_error();
  QUADS_REQUIRE(rows >= 0 && K > 0 && K % 16 == 0, QUADS_ERR_UNSUPPORTED_SHAPE, "K must be a positive multiple of 16");
  QUADS_TRY(validate_groups(group_off, n_groups, rows));
  QUADS_REQUIRE(scale_layout == QUADS_SCALES_LINEAR || scale_layout == QUADS_SCALES_TILED,
                QUADS_ERR_INVALID_ARG, "unknown scale layout %d", scale_layout);
  QUADS_REQUIRE(out_dtype == QUADS_OUT_BF16 || out_dtype == QUADS_OUT_F32, QUADS_ERR_INVALID_ARG,
                "unknown output dtype %d", out_dtype);
  if (rows == 0) return QUADS_OK;
  QUADS_REQUIRE(codes && scales && g && out, QUADS_ERR_INVALID_ARG, "null pointer");
  QUADS_REQUIRE(aligned(codes, 8) && aligned(out, 16), QUADS_ERR_INVALID_ARG,
                "codes must be 8-byte and out 16-byte aligned");
  const int64_t total = rows * (K / 16);
  QUADS_REQUIRE(total < kMaxBlocks, QUADS_ERR_UNSUPPORTED_SHAPE, "tensor above 2^31 blocks of 16");
  size_t smem = group_off ? (static_cast<size_t>(n_groups) + 1) * 4 : 0;
  const uint32_t uniform = group_off ? 1u : static_cast<uint32_t>(rows / n_groups);
  dequant_kernel<<<grid_for(total), kThreads, smem, stream>>>(
      codes, scales, scale_layout, g, group_off, n_groups, make_fastdiv(uniform ? uniform : 1u),
      static_cast<uint32_t>(total), static_cast<uint32_t>(K / 16), make_fastdiv(static_cast<uint32_t>(K / 16)), K,
      out, out_dtype);
  count_launches(1);
  return check_launch("dequant_kernel");
}

size_t quads_channel_scores_workspace_bytes(int64_t rows, int64_t K) {
  if (rows <= 0 || K <= 0) return 256;
  return 256 + static_cast<size_t>(ceil_div(rows, kScoreRows)) * static_cast<size_t>(K) * 4;
}

int quads_channel_scores(const uint16_t* x, int64_t rows, int64_t K, const float* amax_in, float* scores, void* ws,
                         size_t ws_bytes, quads_stream_t stream) {
  clear_error();
  QUADS_TRY(validate_matrix(x, rows, K, K));
  QUADS_REQUIRE(rows > 0, QUADS_ERR_INVALID_ARG, "rows must be > 0");
  QUADS_REQUIRE(scores != nullptr, QUADS_ERR_INVALID_ARG, "scores is null");
  QUADS_REQUIRE(ws && ws_bytes >= quads_channel_scores_workspace_bytes(rows, K), QUADS_ERR_INVALID_ARG,
                "workspace of %zu bytes required", quads_channel_scores_workspace_bytes(rows, K));
  float* amax = static_cast<float*>(ws);
  if (amax_in) {
    if (cudaMemcpyAsync(amax, amax_in, 4, cudaMemcpyDeviceToDevice, stream) != cudaSuccess)
      return set_error(QUADS_ERR_CUDA, "copy of amax failed");
  } else {
    QUADS_TRY(launch_amax(x, rows, K, K, nullptr, 1, amax, stream));
  }
  float* partial = reinterpret_cast<float*>(static_cast<char*>(ws) + 256);
  int64_t n_chunks = ceil_div(rows, kScoreRows);
  int64_t nkb = K / 16;
  dim3 grid(static_cast<unsigned>(ceil_div(nkb, 128)), static_cast<unsigned>(n_chunks));
  channel_partial_kernel<<<grid, 128, 0, stream>>>(x, rows, K, amax, partial);
  count_launches(1);
  QUADS_TRY(check_launch("channel_partial_kernel"));
  channel_reduce_kernel<<<static_cast<unsigned>(ceil_div(K, 256)), 256, 0, stream>>>(partial, n_chunks, K, scores);
  count_launches(1);
  return check_launch("channel_reduce_kernel");
}

int quads_select_channels(const float* scores, int64_t K, int n_sel, int32_t* chan_out, quads_stream_t stream) {
  clear_error();
  QUADS_REQUIRE(scores && chan_out, QUADS_ERR_INVALID_ARG, "null pointer");
  QUADS_REQUIRE(K > 0 && K <= 16384, QUADS_ERR_UNSUPPORTED_SHAPE, "K must be in [1, 16384]");
  QUADS_REQUIRE(n_sel >= 0 && n_sel <= K, QUADS_ERR_INVALID_ARG, "n_sel must be in [0, K]");
  if (n_sel == 0) return QUADS_OK;
  size_t smem = static_cast<size_t>(K) * 4;
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
          cudaSuccess)
    return set_error(QUADS_ERR_CUDA, "cannot raise shared memory of select_kernel");
  select_kernel<<<1, 1024, smem, stream>>>(scores, static_cast<int>(K), n_sel, chan_out);
  count_launches(1);
  return check_launch("select_kernel");
}

}  // extern "C"

namespace quads {
namespace {

int fakequant_impl(const uint16_t* w, int64_t n_mat, int64_t rows, int64_t K, const float* amax_in, int fold_global,
                   uint16_t* w_fq, uint8_t* codes, uint8_t* scales, float* g_out, const int32_t* chan, int n_chan,
                   int chan_raw, uint16_t* w_chan, void* ws, size_t ws_bytes, int64_t ilv_half,
                   quads_stream_t stream) {
  QUADS_REQUIRE(n_mat >= 1 && n_mat <= kMaxGroupsSmem, QUADS_ERR_UNSUPPORTED_SHAPE, "n_mat must be in [1, %d]",
                kMaxGroupsSmem);
  QUADS_TRY(validate_matrix(w, n_mat * rows, K, K));
  QUADS_REQUIRE(rows > 0, QUADS_ERR_INVALID_ARG, "rows must be > 0");
  QUADS_REQUIRE(g_out != nullptr, QUADS_ERR_INVALID_ARG, "g_out is null");
  QUADS_REQUIRE(w_fq == nullptr || aligned(w_fq, 16), QUADS_ERR_INVALID_ARG, "w_fq must be 16-byte aligned");
  QUADS_REQUIRE(codes == nullptr || aligned(codes, 8), QUADS_ERR_INVALID_ARG, "codes must be 8-byte aligned");
  QUADS_REQUIRE(n_chan >= 0 && n_chan <= kMaxChan, QUADS_ERR_UNSUPPORTED_SHAPE, "n_chan must be in [0, %d]",
                kMaxChan);
  QUADS_REQUIRE(n_chan == 0 || (chan && w_chan), QUADS_ERR_INVALID_ARG, "chan and w_chan required with n_chan > 0");
  const float* amax = amax_in;
  if (amax == nullptr) {
    QUADS_REQUIRE(ws && ws_bytes >= quads_quantize_workspace_bytes(static_cast<int>(n_mat)), QUADS_ERR_INVALID_ARG,
                  "workspace of %zu bytes required", quads_quantize_workspace_bytes(static_cast<int>(n_mat)));
    QUADS_TRY(launch_amax(w, n_mat * rows, K, K, nullptr, static_cast<int>(n_mat), static_cast<float*>(ws), stream));
    amax = static_cast<const float*>(ws);
  }
  QuantArgs a{};
  a.x = w; a.rows = n_mat * rows; a.K = K; a.ld = K;
  a.group_off = nullptr; a.n_groups = static_cast<int>(n_mat); a.uniform_rows = rows;
  a.amax = amax; a.codes = codes; a.scales = scales;
  a.scale_layout = (rows % 128 == 0) ? QUADS_SCALES_TILED : QUADS_SCALES_LINEAR;
  a.g_out = g_out; a.chan = chan; a.n_chan = n_chan; a.resid = n_chan ? w_chan : nullptr;
  a.resid_mode = chan_raw ? 2 : 1; a.w_fq = w_fq; a.fold = fold_global ? 1 : 0;
  a.ilv_half = ilv_half;
  return launch_quantize(a, stream);
}

}  // namespace
}  // namespace quads

extern "C" {

int quads_fakequant_weight_ste(const uint16_t* w, int64_t n_mat, int64_t rows, int64_t K, const float* amax_in,
                               int fold_global,
                               uint16_t* w_fq, uint8_t* codes, uint8_t* scales, float* g_out, const int32_t* chan,
                               int n_chan, int chan_raw, uint16_t* w_chan, void* ws, size_t ws_bytes,
                               quads_stream_t stream) {
  clear_error();
  return fakequant_impl(w, n_mat, rows, K, amax_in, fold_global, w_fq, codes, scales, g_out, chan, n_chan, chan_raw,
                        w_chan, ws, ws_bytes, 0, stream);
}

int quads_fakequant_weight_ste_gate_up(const uint16_t* w, int64_t n_mat, int64_t rows, int64_t K,
                                       const float* amax_in, int fold_global, uint16_t* w_fq, uint8_t* codes,
                                       uint8_t* scales, float* g_out, const int32_t* chan, int n_chan, int chan_raw,
                                       uint16_t* w_chan, void* ws, size_t ws_bytes, quads_stream_t stream) {
  clear_error();
  QUADS_REQUIRE(rows > 0 && rows % 128 == 0, QUADS_ERR_UNSUPPORTED_SHAPE,
                "rows (gate and up) must be a positive multiple of 128");
  return fakequant_impl(w, n_mat, rows, K, amax_in, fold_global, w_fq, codes, scales, g_out, chan, n_chan, chan_raw,
                        w_chan, ws, ws_bytes, rows / 2, stream);
}


}  // extern "C"

// ---------------------------------------------------------------------------
// Quantize without any device allocation.
//
// Some callers cannot hand this library a workspace or let it obtain one:
// code whose device memory is entirely owned by another allocator (a
// framework's caching pool, a fixed arena sized once at start-up), plugin
// interfaces that have no way to pass a scratch buffer through, and
// latency-critical loops where an allocation's implicit synchronization is
// not acceptable.  For them, this entry point keeps the only scratch the
// quantizer needs -- one FP32 amax per row group -- in a file-scope device
// array that the module loader places in every GPU's memory when the library
// is loaded and that stays there until the process exits.
//
// The array's name is only a host-side stand-in for the device variable, so
// host code never passes it to a kernel: the device address is obtained with
// cudaGetSymbolAddress on the first call made with a given device and CUDA
// context current, and cached for that device and context.  A call under a
// different context (a non-primary context the caller made current) looks
// the address up again.  cudaDeviceReset destroys the module, and the
// recreated primary context may come back with the same handle, so the
// cached address is not valid across a device reset.  All calls share the array and it keeps the
// last call's contents, so each call clears the part it uses before the amax
// pass; calls that can overlap on the GPU (different streams, or different
// host threads on one device) race on it and must be serialized by the caller.
namespace quads {
namespace {

constexpr int kNoAllocMaxGroups = 1024;                     // 4 KiB of scratch per GPU
static __device__ __align__(256) float g_noalloc_amax[kNoAllocMaxGroups];

struct NoAllocSlot {
  void* ctx;          // CUcontext the address was looked up under
  float* ptr;
};
std::mutex g_noalloc_mutex;
NoAllocSlot g_noalloc_scratch[64] = {};

// The calling thread's current CUDA context, through the driver entry point
// the runtime hands out (no link against the driver library).
int current_context(void** ctx) {
  using GetCtx = int (*)(void**);
  static GetCtx get = nullptr;
  if (get == nullptr) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
      return set_error(QUADS_ERR_CUDA, "cuCtxGetCurrent is not available from the CUDA runtime");
    get = reinterpret_cast<GetCtx>(fn);
  }
  *ctx = nullptr;
  if (get(ctx) != 0 || *ctx == nullptr) return set_error(QUADS_ERR_CUDA, "no current CUDA context");
  return QUADS_OK;
}

int noalloc_scratch(float** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
    return set_error(QUADS_ERR_CUDA, "no usable current CUDA device");
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  NoAllocSlot& slot = g_noalloc_scratch[dev];
  void* ctx = nullptr;
  if (slot.ptr != nullptr) QUADS_TRY(current_context(&ctx));
  if (slot.ptr == nullptr || slot.ctx != ctx) {
    // on a device's first call this also sets up its context, so the handle
    // is read after it
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_amax);
    if (e != cudaSuccess || p == nullptr)
      return set_error(QUADS_ERR_CUDA, "cudaGetSymbolAddress of the quantizer scratch failed: %s",
                       cudaGetErrorString(e));
    QUADS_TRY(current_context(&ctx));
    slot = NoAllocSlot{ctx, static_cast<float*>(p)};
  }
  *out = slot.ptr;
  return QUADS_OK;
}

}  // namespace
}  // namespace quads

extern "C" int quads_quantize_nvfp4_noalloc(const uint16_t* x, int64_t rows, int64_t K, int64_t ld_x,
                                            const int32_t* group_off, int n_groups, const float* amax_in,
                                            uint8_t* codes, uint8_t* scales, int scale_layout, float* g_out,
                                            const int32_t* chan, int n_chan, uint16_t* resid_out,
                                            quads_stream_t stream) {
  clear_error();
  // the scratch's size is this entry point's own limit: checked first, so it
  // holds whatever the general group limit below is
  QUADS_REQUIRE(n_groups <= kNoAllocMaxGroups, QUADS_ERR_UNSUPPORTED_SHAPE,
                "the allocation-free quantizer supports at most %d row groups (got %d)", kNoAllocMaxGroups,
                n_groups);
  QUADS_TRY(validate_matrix(x, rows, K, ld_x));
  QUADS_TRY(validate_groups(group_off, n_groups, rows));
  QUADS_REQUIRE(scale_layout == QUADS_SCALES_LINEAR || scale_layout == QUADS_SCALES_TILED,
                QUADS_ERR_INVALID_ARG, "unknown scale layout %d", scale_layout);
  QUADS_REQUIRE(g_out && (rows == 0 || (codes && scales)), QUADS_ERR_INVALID_ARG,
                "codes, scales and g_out must be non-null (codes and scales may be null for zero rows)");
  QUADS_REQUIRE(aligned(codes, 8), QUADS_ERR_INVALID_ARG, "codes must be 8-byte aligned");
  QUADS_REQUIRE(n_chan >= 0 && n_chan <= kMaxChan, QUADS_ERR_UNSUPPORTED_SHAPE, "n_chan must be in [0, %d]",
                kMaxChan);
  QUADS_REQUIRE(n_chan == 0 || (chan && resid_out), QUADS_ERR_INVALID_ARG,
                "chan and resid_out are required when n_chan > 0");
  if (rows == 0) {
    if (cudaMemsetAsync(g_out, 0, sizeof(float) * n_groups, stream) != cudaSuccess)
      return set_error(QUADS_ERR_CUDA, "memset failed");
    return QUADS_OK;
  }
  const float* amax = amax_in;
  if (amax == nullptr) {
    float* scratch = nullptr;
    QUADS_TRY(noalloc_scratch(&scratch));
    // launch_amax clears scratch[0, n_groups) before accumulating into it
    QUADS_TRY(launch_amax(x, rows, K, ld_x, group_off, n_groups, scratch, stream));
    amax = scratch;
  }
  QuantArgs a{};
  a.x = x; a.rows = rows; a.K = K; a.ld = ld_x;
  a.group_off = group_off; a.n_groups = n_groups; a.uniform_rows = group_off ? 1 : rows / n_groups;
  a.amax = amax; a.codes = codes; a.scales = scales; a.scale_layout = scale_layout; a.g_out = g_out;
  a.chan = chan; a.n_chan = n_chan; a.resid = n_chan ? resid_out : nullptr; a.resid_mode = 0;
  a.w_fq = nullptr; a.fold = 1;
  return launch_quantize(a, stream);
}
