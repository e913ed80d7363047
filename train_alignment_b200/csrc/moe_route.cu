// MoE routing kernels: top-k router, stable expert permutation (histogram,
// scan, in-order ranking with warp match/ballot), gather of the quantized rows
// into expert order, SwiGLU with per-expert amax, and the weighted combine.
//
// Method: experts are chosen discretely by the router ([TRACE]
// "Fonctionnement"); the expert layer is an NVFP4 W4A4 MoE ([QUADS-fr §1]).
// The permutation is a plain stable counting sort: no atomics decide a
// position, so expert_off, row_of and src_of are bit-identical run to run.
#include "common.cuh"

namespace quads {
namespace {

constexpr int kMaxE = 256;
constexpr int kMaxK = 8;
constexpr int kChunk = 4096;          // (token, slot) pairs per permutation chunk
constexpr int kRankThreads = 256;

// -------------------------------------------------------------------- router

// One warp per token. Each lane holds logits e = lane + 32 i.
__global__ void __launch_bounds__(256) router_kernel(const float* __restrict__ logits, int64_t T, int E, int k,
                                                     int renorm, int32_t* __restrict__ idx_out,
                                                     float* __restrict__ w_out) {
  const int lane = threadIdx.x & 31;
  const int64_t t = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (t >= T) return;
  constexpr int kPer = kMaxE / 32;
  float v[kPer];
  const float* row = logits + t * E;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    int e = lane + 32 * i;
    v[i] = (e < E) ? row[e] : -INFINITY;
  }
  unsigned int taken = 0u;      // bit i: my slot i already selected
  float sel_v[kMaxK];
  int sel_e[kMaxK];
  for (int s = 0; s < k; ++s) {
    // local best among my unselected entries: larger value, then lower index
    float bv = -INFINITY;
    int be = 0x7FFFFFFF;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      int e = lane + 32 * i;
      if (e < E && !((taken >> i) & 1u) && (v[i] > bv || (v[i] == bv && e < be))) { bv = v[i]; be = e; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (ov > bv || (ov == bv && oe < be)) { bv = ov; be = oe; }
    }
    sel_v[s] = bv;
    sel_e[s] = be;
    if ((be & 31) == lane) taken |= 1u << (be >> 5);
  }
  // softmax weights
  float m, z = 0.0f;
  if (renorm) {
    m = sel_v[0];                                   // the first selected is the max
    for (int s = 0; s < k; ++s) z += expf(sel_v[s] - m);
  } else {
    m = sel_v[0];
#pragma unroll
    for (int i = 0; i < kPer; ++i)
      if (lane + 32 * i < E) z += expf(v[i] - m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
  }
  if (lane < k) {
    float ev = 0.0f;
    int ee = 0;
    for (int s = 0; s < k; ++s)
      if (s == lane) { ev = sel_v[s]; ee = sel_e[s]; }
    idx_out[t * k + lane] = ee;
    w_out[t * k + lane] = expf(ev - m) / z;
  }
}

// --------------------------------------------------------------- permutation

// cnt[chunk][e]: pairs of expert e in the chunk.
__global__ void __launch_bounds__(256) hist_kernel(const int32_t* __restrict__ idx, int64_t n_pairs, int E,
                                                   int32_t* __restrict__ cnt) {
  __shared__ int32_t h[kMaxE];
  for (int i = threadIdx.x; i < E; i += blockDim.x) h[i] = 0;
  __syncthreads();
  const int64_t lo = static_cast<int64_t>(blockIdx.x) * kChunk;
  const int64_t hi = min(n_pairs, lo + kChunk);
  for (int64_t i = lo + threadIdx.x; i < hi; i += blockDim.x) {
    int e = idx[i];
    if (e >= 0 && e < E) atomicAdd(&h[e], 1);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < E; i += blockDim.x) cnt[static_cast<int64_t>(blockIdx.x) * E + i] = h[i];
}

// One block, one thread per expert: totals, 128-padded offsets, per-chunk
// bases, and -1 in the pad rows of every expert's segment.
__global__ void __launch_bounds__(kMaxE) scan_kernel(const int32_t* __restrict__ cnt, int n_chunks, int E,
                                                     int32_t* __restrict__ base, int32_t* __restrict__ expert_off,
                                                     int32_t* __restrict__ src_of) {
  __shared__ int32_t padded[kMaxE + 1];
  const int e = threadIdx.x;
  int total = 0;
  if (e < E)
    for (int c = 0; c < n_chunks; ++c) total += cnt[c * E + e];
  padded[e] = (e < E) ? (total + 127) / 128 * 128 : 0;
  __syncthreads();
  // exclusive scan over experts (E <= 256, done serially per thread for clarity and determinism)
  int off = 0;
  for (int j = 0; j < e && j < E; ++j) off += padded[j];
  if (e < E) {
    expert_off[e] = off;
    int run = off;
    for (int c = 0; c < n_chunks; ++c) {
      base[c * E + e] = run;
      run += cnt[c * E + e];
    }
    for (int r = off + total; r < off + padded[e]; ++r) src_of[r] = -1;
    if (e == E - 1) expert_off[E] = off + padded[e];
  }
}

// Ranks the chunk's pairs in order: rounds of 256 pairs, within a warp by
// __match_any_sync, across warps by per-warp counts, across rounds by a
// running count per expert.
__global__ void __launch_bounds__(kRankThreads) rank_kernel(const int32_t* __restrict__ idx, int64_t n_pairs, int k,
                                                            int E, const int32_t* __restrict__ base,
                                                            int32_t* __restrict__ row_of, int32_t* __restrict__ src_of) {
  constexpr int kWarps = kRankThreads / 32;
  __shared__ int32_t running[kMaxE];
  __shared__ int32_t wcnt[kWarps][kMaxE];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < E; i += blockDim.x) running[i] = base[static_cast<int64_t>(blockIdx.x) * E + i];
  const int64_t lo = static_cast<int64_t>(blockIdx.x) * kChunk;
  const int64_t hi = min(n_pairs, lo + kChunk);
  for (int64_t r0 = lo; r0 < hi; r0 += kRankThreads) {
    for (int i = threadIdx.x; i < kWarps * kMaxE; i += blockDim.x) (&wcnt[0][0])[i] = 0;
    __syncthreads();
    const int64_t i = r0 + threadIdx.x;
    const bool valid = i < hi;
    const int e = valid ? idx[i] : -1;
    const unsigned int peers = __match_any_sync(0xffffffffu, e);
    const int rank_w = __popc(peers & ((1u << lane) - 1u));
    const int leader = __ffs(peers) - 1;
    if (valid && lane == leader && e >= 0 && e < E) wcnt[wid][e] = __popc(peers);
    __syncthreads();
    if (valid && e >= 0 && e < E) {
      int pos = running[e] + rank_w;
      for (int w = 0; w < wid; ++w) pos += wcnt[w][e];
      row_of[i] = pos;
      src_of[pos] = static_cast<int32_t>(i / k);
    }
    __syncthreads();
    for (int x = threadIdx.x; x < E; x += blockDim.x) {
      int add = 0;
      for (int w = 0; w < kWarps; ++w) add += wcnt[w][x];
      running[x] += add;
    }
    __syncthreads();
  }
}

// Whole permutation in one block for small batches (<= kSmallPairs pairs):
// histogram, padded offsets, pad rows and the in-order ranking.
constexpr int kSmallThreads = 1024;
constexpr int kSmallWarps = kSmallThreads / 32;
constexpr int kSmallPairs = kSmallThreads * 32;   // 32768: up to 32 pairs per lane

// The whole permutation in one CTA for up to 32768 routed pairs.  Warp w owns
// the contiguous pairs [w P, (w + 1) P) (P a multiple of 32), held in
// registers (the expert of pair w P + 32 j + lane as 16 bits), read from
// global memory once:
//   1. per-warp expert histogram: one shared-memory add per distinct expert
//      among the 32 lanes (__match_any_sync), warp-synchronous;
//   2. per expert, the exclusive prefix over warps (one thread per expert),
//      and the 128-padded expert offsets (a warp-shuffle scan);
//   3. stable ranks: pair i of expert e goes to offset(e) + #(earlier pairs
//      of e in earlier warps) + #(earlier pairs of e in this warp).
// Padding rows of every expert segment get src_of = -1.
// kPerLane: pairs per lane (4 or 32; the small variant keeps the unrolled
// loops short enough to stay in the instruction cache).
template <int kPerLane>
__global__ void __launch_bounds__(kSmallThreads) permute_small_kernel(const int32_t* __restrict__ idx,
                                                                      int n_pairs, int k, int E,
                                                                      int32_t* __restrict__ expert_off,
                                                                      int32_t* __restrict__ row_of,
                                                                      int32_t* __restrict__ src_of) {
  __shared__ int32_t wbase[kSmallWarps * kMaxE];        // [warp][expert]: count, then first row
  __shared__ int32_t cnt_s[kMaxE];
  __shared__ int32_t off_s[kMaxE + 1];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int per_warp = ((n_pairs + kSmallWarps - 1) / kSmallWarps + 31) & ~31;
  const int J = per_warp / 32;                          // <= kPerLane
  const int w0 = wid * per_warp;
  // expert of pair j of this lane as 16 bits (-1: no pair / out of range), two per register
  uint32_t vp[kPerLane / 2];
#pragma unroll
  for (int j = 0; j < kPerLane; j += 2) {
    int e2[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int i = w0 + (j + u) * 32 + lane;
      const int e = (j + u < J && i < n_pairs) ? __ldg(idx + i) : -1;
      e2[u] = (e >= 0 && e < E) ? e : -1;
    }
    vp[j / 2] = (static_cast<uint32_t>(e2[0]) & 0xFFFFu) | (static_cast<uint32_t>(e2[1]) << 16);
  }
  auto v_of = [&](int j) { return static_cast<int>(static_cast<int16_t>(vp[j >> 1] >> (16 * (j & 1)))); };
  for (int i = threadIdx.x; i < kSmallWarps * E; i += blockDim.x) wbase[i] = 0;
  __syncthreads();
  // 1. per-warp histogram
#pragma unroll
  for (int j = 0; j < kPerLane; ++j) {
    if (j < J) {                                        // warp-uniform
      const int e = v_of(j);
      const unsigned int peers = __match_any_sync(0xffffffffu, e);
      if (e >= 0 && lane == __ffs(peers) - 1) wbase[wid * E + e] += __popc(peers);
      __syncwarp();
    }
  }
  __syncthreads();
  // 2a. per expert: exclusive prefix over warps, total count
  if (threadIdx.x < E) {
    const int e = threadIdx.x;
    int run = 0;
    for (int w = 0; w < kSmallWarps; ++w) {
      const int c = wbase[w * E + e];
      wbase[w * E + e] = run;
      run += c;
    }
    cnt_s[e] = run;
  }
  __syncthreads();
  // 2b. expert offsets: exclusive scan of the 128-padded counts (8 experts per lane)
  if (wid == 0) {
    int loc[8], sum = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int e = lane * 8 + q;
      loc[q] = sum;
      sum += (e < E) ? (cnt_s[e] + 127) / 128 * 128 : 0;
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
#pragma unroll
    for (int q = 0; q < 8; ++q)
      if (lane * 8 + q < E) off_s[lane * 8 + q] = incl - sum + loc[q];
    if (lane == 31) off_s[E] = incl;
  }
  __syncthreads();
  const int total_rows = off_s[E];
  for (int i = threadIdx.x; i <= E; i += blockDim.x) expert_off[i] = off_s[i];
  for (int r = threadIdx.x; r < total_rows; r += blockDim.x) src_of[r] = -1;   // overwritten below for real rows
  for (int i = threadIdx.x; i < kSmallWarps * E; i += blockDim.x) wbase[i] += off_s[i % E];
  __syncthreads();                                      // also orders the -1 fill before the row writes
  // 3. stable ranks
  const unsigned int lt = (1u << lane) - 1u;
#pragma unroll
  for (int j = 0; j < kPerLane; ++j) {
    if (j < J) {                                        // warp-uniform
      const int e = v_of(j);
      const unsigned int peers = __match_any_sync(0xffffffffu, e);
      if (e >= 0) {
        const int i = w0 + j * 32 + lane;
        const int pos = wbase[wid * E + e] + __popc(peers & lt);
        row_of[i] = pos;
        src_of[pos] = i / k;
      }
      __syncwarp();
      if (e >= 0 && lane == __ffs(peers) - 1) wbase[wid * E + e] += __popc(peers);
      __syncwarp();
    }
  }
}

// ------------------------------------------------------------------- gather

// One warp per expert-ordered row p < expert_off[E].
__global__ void __launch_bounds__(256) gather_kernel(const int32_t* __restrict__ src_of,
                                                     const int32_t* __restrict__ expert_off, int E, int64_t rows_cap,
                                                     const uint8_t* __restrict__ a_codes,
                                                     const uint8_t* __restrict__ a_scales, int64_t K,
                                                     const uint16_t* __restrict__ a_resid, int n_chan,
                                                     uint8_t* __restrict__ pa_codes, uint8_t* __restrict__ pa_scales,
                                                     uint16_t* __restrict__ pa_resid) {
  const int lane = threadIdx.x & 31;
  const int64_t rows = expert_off[E];
  const int64_t nkb = K / 16, ncol_tiles = nkb / 4;
  const int64_t cbytes = K / 2, ncv = cbytes / 16;
  // residual rows in 16-byte vectors when they are whole and aligned
  const bool rvec = n_chan % 8 == 0 && (reinterpret_cast<uintptr_t>(a_resid) & 15) == 0 &&
                    (reinterpret_cast<uintptr_t>(pa_resid) & 15) == 0;
  for (int64_t p = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; p < rows;
       p += (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5) {
    const int t = src_of[p];
    const bool has = t >= 0;
    // codes: 16-byte vectors, four loads in flight per lane before the stores
    uint4* dc = reinterpret_cast<uint4*>(pa_codes + p * cbytes);
    const uint4* sc = reinterpret_cast<const uint4*>(a_codes + static_cast<int64_t>(t) * cbytes);
    for (int64_t j0 = lane; j0 < ncv; j0 += 128) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t j = j0 + 32 * u;
        v[u] = (has && j < ncv) ? __ldg(sc + j) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (j0 + 32 * u < ncv) dc[j0 + 32 * u] = v[u];
    }
    // scales: 4 consecutive blocks are 4 contiguous bytes in both layouts
    for (int64_t q = lane; q < nkb / 4; q += 32) {
      uint32_t v = has ? __ldg(reinterpret_cast<const uint32_t*>(a_scales + static_cast<int64_t>(t) * nkb) + q) : 0u;
      *reinterpret_cast<uint32_t*>(pa_scales + tiled_scale_offset(p, 4 * q, ncol_tiles)) = v;
    }
    if (n_chan) {
      if (rvec) {
        const int nrv = n_chan / 8;
        const uint4* sr = reinterpret_cast<const uint4*>(a_resid + static_cast<int64_t>(t) * n_chan);
        uint4* dr = reinterpret_cast<uint4*>(pa_resid + p * n_chan);
        for (int j = lane; j < nrv; j += 32) dr[j] = has ? __ldg(sr + j) : make_uint4(0, 0, 0, 0);
      } else {
        for (int j = lane; j < n_chan; j += 32)
          pa_resid[p * n_chan + j] = has ? a_resid[static_cast<int64_t>(t) * n_chan + j] : 0;
      }
    }
  }
}

// One warp per expert-ordered row: the BF16 row of its token in 16-byte
// vectors, or zeros on a pad row (the trainer's BF16 activations gathered for
// the W4A16 GEMMs).
__global__ void __launch_bounds__(256) gather_bf16_kernel(const int32_t* __restrict__ src_of,
                                                          const int32_t* __restrict__ expert_off, int E,
                                                          const uint16_t* __restrict__ x, int64_t H,
                                                          uint16_t* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int64_t rows = expert_off[E];
  const int64_t nvec = H / 8;
  for (int64_t p = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; p < rows;
       p += (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5) {
    const int t = src_of[p];
    const bool has = t >= 0;
    uint4* d = reinterpret_cast<uint4*>(out + p * H);
    const uint4* sx = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(t) * H);
    for (int64_t j0 = lane; j0 < nvec; j0 += 128) {     // four loads in flight per lane
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t j = j0 + 32 * u;
        v[u] = (has && j < nvec) ? __ldg(sx + j) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (j0 + 32 * u < nvec) d[j0 + 32 * u] = v[u];
    }
  }
}

// ------------------------------------------------------------------- SwiGLU

// Each thread: 8 outputs of one row.  Per-expert amax via shared atomics.
__global__ void __launch_bounds__(256) swiglu_kernel(const uint16_t* __restrict__ y, int64_t F,
                                                     const int32_t* __restrict__ expert_off, int E,
                                                     uint16_t* __restrict__ h, unsigned int* __restrict__ amax_bits) {
  __shared__ int32_t off_s[kMaxE + 1];
  __shared__ unsigned int am_s[kMaxE];
  for (int i = threadIdx.x; i <= E; i += blockDim.x) {
    off_s[i] = expert_off[i];
    if (i < E) am_s[i] = 0u;
  }
  __syncthreads();
  RowGroups grp{off_s, E, FastDiv{1u, 1u, 0u}};
  const int64_t rows = off_s[E];
  const int64_t per_row = F / 8;
  const int64_t total = rows * per_row;
  for (int64_t b = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; b < total;
       b += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = b / per_row, c8 = b - row * per_row;
    const uint4 gv = __ldg(reinterpret_cast<const uint4*>(y + row * 2 * F + c8 * 8));
    const uint4 uv = __ldg(reinterpret_cast<const uint4*>(y + row * 2 * F + F + c8 * 8));
    const uint32_t* gp = reinterpret_cast<const uint32_t*>(&gv);
    const uint32_t* up = reinterpret_cast<const uint32_t*>(&uv);
    uint32_t o[4];
    unsigned int m = 0u;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float r[2];
#pragma unroll
      for (int hl = 0; hl < 2; ++hl) {
        float gt = bf16_bits_to_float(hl ? (gp[j] >> 16) : (gp[j] & 0xFFFFu));
        float ut = bf16_bits_to_float(hl ? (up[j] >> 16) : (up[j] & 0xFFFFu));
        float sg = __fdividef(gt, 1.0f + __expf(-gt));   // relative error ~1e-6, far below BF16 rounding
        r[hl] = __fmul_rn(sg, ut);
      }
      o[j] = pack_bf16x2(r[0], r[1]);
      m = max(m, o[j] & 0x7FFFu);
      m = max(m, (o[j] >> 16) & 0x7FFFu);
    }
    *reinterpret_cast<uint4*>(h + row * F + c8 * 8) = make_uint4(o[0], o[1], o[2], o[3]);
    if (amax_bits && m) atomicMax(&am_s[grp.of(row)], m);
  }
  __syncthreads();
  if (amax_bits)
    for (int i = threadIdx.x; i < E; i += blockDim.x)
      if (am_s[i]) atomicMax(&amax_bits[i], am_s[i] << 16);
}

// ------------------------------------------------------------------ combine

// One warp per token; each lane 8 consecutive outputs per step.
__global__ void __launch_bounds__(256) combine_kernel(const uint16_t* __restrict__ y, const int32_t* __restrict__ row_of,
                                                      const float* __restrict__ w, int64_t T, int k, int64_t H,
                                                      uint16_t* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int64_t t = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (t >= T) return;
  int rows[kMaxK];
  float ws[kMaxK];
  for (int s = 0; s < k; ++s) {
    rows[s] = row_of[t * k + s];
    ws[s] = w[t * k + s];
  }
  // two 8-column chunks per lane per iteration, the loads of all k slots for
  // both issued before any is used (up to 16 independent 16-byte loads)
  for (int64_t c0 = lane * 8; c0 < H; c0 += 2 * 32 * 8) {
    uint4 v[kMaxK][2];
#pragma unroll
    for (int s = 0; s < kMaxK; ++s) {
      if (s < k) {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int64_t c = c0 + u * 256;
          v[s][u] = c < H ? __ldg(reinterpret_cast<const uint4*>(y + static_cast<int64_t>(rows[s]) * H + c))
                          : make_uint4(0, 0, 0, 0);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int64_t c = c0 + u * 256;
      float acc[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[j] = 0.0f;
#pragma unroll
      for (int s = 0; s < kMaxK; ++s) {
        if (s < k) {
          const uint32_t* p = reinterpret_cast<const uint32_t*>(&v[s][u]);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            acc[2 * j] = __fmaf_rn(ws[s], bf16_bits_to_float(p[j] & 0xFFFFu), acc[2 * j]);
            acc[2 * j + 1] = __fmaf_rn(ws[s], bf16_bits_to_float(p[j] >> 16), acc[2 * j + 1]);
          }
        }
      }
      if (c < H)
        *reinterpret_cast<uint4*>(out + t * H + c) =
            make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]), pack_bf16x2(acc[4], acc[5]),
                       pack_bf16x2(acc[6], acc[7]));
    }
  }
}

int grid_rows(int64_t work_items, int per_block) {
  int64_t g = ceil_div(work_items, per_block);
  int64_t cap = static_cast<int64_t>(num_sms()) * 16;
  if (g > cap) g = cap;
  return static_cast<int>(g < 1 ? 1 : g);
}

}  // namespace
}  // namespace quads

using namespace quads;

extern "C" {

int64_t quads_moe_rows_capacity(int64_t T, int k, int E) {
  if (T < 0 || k <= 0 || E <= 0) return 0;
  return (ceil_div(T * k, 128) + E) * 128;
}

size_t quads_moe_permute_workspace_bytes(int64_t T, int k, int E) {
  if (T < 0 || k <= 0 || E <= 0) return 0;
  int64_t n_chunks = ceil_div(T * k, kChunk);
  if (n_chunks < 1) n_chunks = 1;
  return static_cast<size_t>(2 * n_chunks * E * 4 + 256);
}

int quads_moe_router_topk(const float* logits, int64_t T, int E, int k, int renorm, int32_t* topk_idx,
                          float* topk_w, quads_stream_t stream) {
  clear_error();
  QUADS_REQUIRE(T >= 0, QUADS_ERR_INVALID_ARG, "T must be >= 0");
  QUADS_REQUIRE(E >= 1 && E <= kMaxE, QUADS_ERR_UNSUPPORTED_SHAPE, "E must be in [1, %d]", kMaxE);
  QUADS_REQUIRE(k >= 1 && k <= kMaxK && k <= E, QUADS_ERR_UNSUPPORTED_SHAPE, "k must be in [1, min(E, %d)]", kMaxK);
  if (T == 0) return QUADS_OK;
  QUADS_REQUIRE(logits && topk_idx && topk_w, QUADS_ERR_INVALID_ARG, "null pointer");
  router_kernel<<<static_cast<unsigned>(ceil_div(T * 32, 256)), 256, 0, stream>>>(logits, T, E, k, renorm ? 1 : 0,
                                                                                 topk_idx, topk_w);
  count_launches(1);
  return check_launch("router_kernel");
}

int quads_moe_permute(const int32_t* topk_idx, int64_t T, int k, int E, int32_t* expert_off, int32_t* row_of,
                      int32_t* src_of, void* ws, size_t ws_bytes, quads_stream_t stream) {
  clear_error();
  QUADS_REQUIRE(T >= 0, QUADS_ERR_INVALID_ARG, "T must be >= 0");
  QUADS_REQUIRE(E >= 1 && E <= kMaxE, QUADS_ERR_UNSUPPORTED_SHAPE, "E must be in [1, %d]", kMaxE);
  QUADS_REQUIRE(k >= 1 && k <= kMaxK, QUADS_ERR_UNSUPPORTED_SHAPE, "k must be in [1, %d]", kMaxK);
  QUADS_REQUIRE(T * k < (int64_t(1) << 30), QUADS_ERR_UNSUPPORTED_SHAPE, "T * k too large");
  QUADS_REQUIRE(expert_off && src_of && (T == 0 || (topk_idx && row_of)), QUADS_ERR_INVALID_ARG, "null pointer");
  QUADS_REQUIRE(ws && ws_bytes >= quads_moe_permute_workspace_bytes(T, k, E), QUADS_ERR_INVALID_ARG,
                "workspace of %zu bytes required", quads_moe_permute_workspace_bytes(T, k, E));
  const int64_t n_pairs = T * k;
  if (n_pairs <= kSmallPairs) {
    if (n_pairs <= kSmallThreads * 4)
      permute_small_kernel<4><<<1, kSmallThreads, 0, stream>>>(topk_idx, static_cast<int>(n_pairs), k, E,
                                                               expert_off, row_of, src_of);
    else
      permute_small_kernel<32><<<1, kSmallThreads, 0, stream>>>(topk_idx, static_cast<int>(n_pairs), k, E,
                                                                expert_off, row_of, src_of);
    count_launches(1);
    return check_launch("permute_small_kernel");
  }
  int n_chunks = static_cast<int>(ceil_div(n_pairs, kChunk));
  if (n_chunks < 1) n_chunks = 1;
  int32_t* cnt = static_cast<int32_t*>(ws);
  int32_t* base = cnt + static_cast<int64_t>(n_chunks) * E;
  hist_kernel<<<n_chunks, 256, 0, stream>>>(topk_idx, n_pairs, E, cnt);
  count_launches(1);
  QUADS_TRY(check_launch("hist_kernel"));
  scan_kernel<<<1, kMaxE, 0, stream>>>(cnt, n_chunks, E, base, expert_off, src_of);
  count_launches(1);
  QUADS_TRY(check_launch("scan_kernel"));
  if (n_pairs == 0) return QUADS_OK;
  rank_kernel<<<n_chunks, kRankThreads, 0, stream>>>(topk_idx, n_pairs, k, E, base, row_of, src_of);
  count_launches(1);
  return check_launch("rank_kernel");
}

int quads_moe_gather(const int32_t* src_of, const int32_t* expert_off, int E, int64_t rows_cap,
                     const uint8_t* a_codes, const uint8_t* a_scales, int64_t K, const uint16_t* a_resid, int n_chan,
                     uint8_t* pa_codes, uint8_t* pa_scales, uint16_t* pa_resid, quads_stream_t stream) {
  clear_error();
  QUADS_REQUIRE(E >= 1 && E <= kMaxE, QUADS_ERR_UNSUPPORTED_SHAPE, "E must be in [1, %d]", kMaxE);
  QUADS_REQUIRE(K > 0 && K % 64 == 0, QUADS_ERR_UNSUPPORTED_SHAPE, "K must be a positive multiple of 64");
  QUADS_REQUIRE(rows_cap >= 0 && rows_cap % 128 == 0, QUADS_ERR_INVALID_ARG, "rows_cap must be a multiple of 128");
  QUADS_REQUIRE(n_chan >= 0 && n_chan <= 256, QUADS_ERR_UNSUPPORTED_SHAPE, "n_chan must be in [0, 256]");
  QUADS_REQUIRE(src_of && expert_off && a_codes && a_scales && pa_codes && pa_scales, QUADS_ERR_INVALID_ARG,
                "null pointer");
  QUADS_REQUIRE(n_chan == 0 || (a_resid && pa_resid), QUADS_ERR_INVALID_ARG, "residual pointers required");
  QUADS_REQUIRE(aligned(a_codes, 16) && aligned(pa_codes, 16) && aligned(a_scales, 4) && aligned(pa_scales, 4),
                QUADS_ERR_INVALID_ARG, "codes must be 16-byte and scales 4-byte aligned");
  if (rows_cap == 0) return QUADS_OK;
  gather_kernel<<<grid_rows(rows_cap * 32, 256), 256, 0, stream>>>(src_of, expert_off, E, rows_cap, a_codes,
                                                                    a_scales, K, a_resid, n_chan, pa_codes,
                                                                    pa_scales, pa_resid);
  count_launches(1);
  return check_launch("gather_kernel");
}

int quads_moe_gather_bf16(const int32_t* src_of, const int32_t* expert_off, int E, int64_t rows_cap,
                          const uint16_t* x, int64_t H, uint16_t* out, quads_stream_t stream) {
  clear_error();
  QUADS_REQUIRE(E >= 1 && E <= kMaxE, QUADS_ERR_UNSUPPORTED_SHAPE, "E must be in [1, %d]", kMaxE);
  QUADS_REQUIRE(H > 0 && H % 8 == 0, QUADS_ERR_UNSUPPORTED_SHAPE, "H must be a positive multiple of 8");
  QUADS_REQUIRE(rows_cap >= 0 && rows_cap % 128 == 0, QUADS_ERR_INVALID_ARG, "rows_cap must be a multiple of 128");
  QUADS_REQUIRE(src_of && expert_off && x && out, QUADS_ERR_INVALID_ARG, "null pointer");
  QUADS_REQUIRE(aligned(x, 16) && aligned(out, 16), QUADS_ERR_INVALID_ARG, "x and out must be 16-byte aligned");
  if (rows_cap == 0) return QUADS_OK;
  gather_bf16_kernel<<<grid_rows(rows_cap * 32, 256), 256, 0, stream>>>(src_of, expert_off, E, x, H, out);
  count_launches(1);
  return check_launch("gather_bf16_kernel");
}

int quads_moe_route_permute(const float* logits, int64_t T, int E, int k, int renorm, int32_t* topk_idx,
                            float* topk_w, int32_t* expert_off, int32_t* row_of, int32_t* src_of, int64_t rows_cap,
                            const uint8_t* a_codes, const uint8_t* a_scales, int64_t K, const uint16_t* a_resid,
                            int n_chan, uint8_t* pa_codes, uint8_t* pa_scales, uint16_t* pa_resid, void* ws,
                            size_t ws_bytes, quads_stream_t stream) {
  QUADS_TRY(quads_moe_router_topk(logits, T, E, k, renorm, topk_idx, topk_w, stream));
  QUADS_TRY(quads_moe_permute(topk_idx, T, k, E, expert_off, row_of, src_of, ws, ws_bytes, stream));
  return quads_moe_gather(src_of, expert_off, E, rows_cap, a_codes, a_scales, K, a_resid, n_chan, pa_codes,
                          pa_scales, pa_resid, stream);
}

int quads_swiglu(const uint16_t* y, int64_t rows_cap, int64_t F, const int32_t* expert_off, int E, uint16_t* h,
                 float* amax_out, quads_stream_t stream) {
  clear_error();
  QUADS_REQUIRE(F > 0 && F % 8 == 0, QUADS_ERR_UNSUPPORTED_SHAPE, "F must be a positive multiple of 8");
  QUADS_REQUIRE(E >= 1 && E <= kMaxE, QUADS_ERR_UNSUPPORTED_SHAPE, "E must be in [1, %d]", kMaxE);
  QUADS_REQUIRE(rows_cap >= 0, QUADS_ERR_INVALID_ARG, "rows_cap must be >= 0");
  QUADS_REQUIRE(y && h && expert_off && aligned(y, 16) && aligned(h, 16), QUADS_ERR_INVALID_ARG,
                "y and h must be non-null and 16-byte aligned");
  if (amax_out && cudaMemsetAsync(amax_out, 0, sizeof(float) * E, stream) != cudaSuccess)
    return set_error(QUADS_ERR_CUDA, "memset of amax_out failed");
  if (rows_cap == 0) return QUADS_OK;
  swiglu_kernel<<<grid_rows(rows_cap * (F / 8), 256), 256, 0, stream>>>(
      y, F, expert_off, E, h, reinterpret_cast<unsigned int*>(amax_out));
  count_launches(1);
  return check_launch("swiglu_kernel");
}

int quads_moe_unpermute_combine(const uint16_t* y, const int32_t* row_of, const float* topk_w, int64_t T, int k,
                                int64_t H, uint16_t* out, quads_stream_t stream) {
  clear_error();
  QUADS_REQUIRE(T >= 0 && H > 0 && H % 8 == 0, QUADS_ERR_UNSUPPORTED_SHAPE, "H must be a positive multiple of 8");
  QUADS_REQUIRE(k >= 1 && k <= kMaxK, QUADS_ERR_UNSUPPORTED_SHAPE, "k must be in [1, %d]", kMaxK);
  if (T == 0) return QUADS_OK;
  QUADS_REQUIRE(y && row_of && topk_w && out && aligned(y, 16) && aligned(out, 16), QUADS_ERR_INVALID_ARG,
                "null or misaligned pointer");
  combine_kernel<<<static_cast<unsigned>(ceil_div(T * 32, 256)), 256, 0, stream>>>(y, row_of, topk_w, T, k, H, out);
  count_launches(1);
  return check_launch("combine_kernel");
}

}  // extern "C"
