// TRACE record: the rollout's export of its quantization results for a deep
// layer, and the trainer's replay of them.
//
// Method: [TRACE] "L'idée centrale de TRACE" -- the rollout's quantization
// results guide the trainer's rounding; a compact cache keeps the mantissa and
// the scale factors of the deep layers.  [TRACE] "Fonctionnement" -- the
// rollout quantizes and records, the trainer reads the record during its
// forward pass.  [TRACE] "Impact" -- the engine exports, the trainer consumes.
//
// Export is a multi-segment device copy (HBM-bound, 16-byte vectors).  Replay
// is one pass that reads the recorded codes and scales, writes the replayed
// operand and, given the trainer's own activation, counts the codes and
// scales its own rounding would have chosen differently.
#include <cstring>

#include "trace_common.cuh"

namespace quads {
namespace {

constexpr int kMaxSegments = 16;
constexpr int kThreads = 256;

struct Segment {
  const uint8_t* src;
  uint64_t dst_off;
  uint64_t bytes;
};

struct ExportArgs {
  Segment seg[kMaxSegments];
  int n_seg;
  trace_qrecord_header hdr;
};

__global__ void __launch_bounds__(kThreads) export_kernel(ExportArgs a, uint8_t* __restrict__ record) {
  const int si = blockIdx.y;
  if (si == 0 && blockIdx.x == 0) {
    const uint8_t* h = reinterpret_cast<const uint8_t*>(&a.hdr);
    for (int i = threadIdx.x; i < static_cast<int>(sizeof(trace_qrecord_header)); i += blockDim.x) record[i] = h[i];
  }
  if (si >= a.n_seg) return;
  const Segment s = a.seg[si];
  uint8_t* dst = record + s.dst_off;
  const uint64_t tid = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const uint64_t stride = static_cast<uint64_t>(gridDim.x) * blockDim.x;
  uint64_t head = 0;
  if ((reinterpret_cast<uintptr_t>(s.src) & 15u) == 0) {
    const uint64_t nv = s.bytes / 16;
    const uint4* src4 = reinterpret_cast<const uint4*>(s.src);
    uint4* dst4 = reinterpret_cast<uint4*>(dst);
    for (uint64_t i = tid; i < nv; i += stride) dst4[i] = __ldg(src4 + i);
    head = nv * 16;
  }
  for (uint64_t i = head + tid; i < s.bytes; i += stride) dst[i] = s.src[i];
}

uint64_t align256(uint64_t v) { return (v + 255) & ~uint64_t(255); }

// ------------------------------------------------------------------- replay

struct ReplayArgs {
  const uint8_t* record;
  uint64_t record_bytes;
  int layer_id, which;
  int64_t rows, K;
  const uint16_t* x_train;
  uint16_t* x_hat;
  unsigned long long* counts;
  int32_t* status;
  FastDiv nkb_div;         // K / 16 (checked against the record on the device)
};

__device__ bool record_ok(const ReplayArgs& a, const trace_qrecord_header& h) {
  if (h.magic != TRACE_QRECORD_MAGIC || h.version != TRACE_QRECORD_VERSION) return false;
  if (h.layer_id != a.layer_id || h.total_bytes > a.record_bytes) return false;
  if (a.which < 0 || a.which >= TRACE_MAX_TENSORS) return false;
  const trace_qtensor_desc& d = h.t[a.which];
  if (!d.present || d.rows != a.rows || d.K != a.K) return false;
  if (d.K <= 0 || d.K % 16 != 0 || d.K > 65536 || d.rows < 0) return false;
  if (d.rows * (d.K / 16) >= (int64_t(1) << 31)) return false;
  if (d.n_groups < 1 || d.n_groups > 1024 || d.n_chan < 0 || d.n_chan > 256) return false;
  if (d.scale_layout != QUADS_SCALES_LINEAR && d.scale_layout != QUADS_SCALES_TILED) return false;
  const uint64_t cb = static_cast<uint64_t>(d.rows) * (d.K / 2);
  const uint64_t sb = static_cast<uint64_t>(scale_bytes(d.rows, d.K, d.scale_layout));
  if (d.codes_bytes != cb || d.scales_bytes != sb) return false;
  auto inside = [&](uint64_t off, uint64_t bytes) { return off % 16 == 0 && off <= h.total_bytes && bytes <= h.total_bytes - off; };
  if (!inside(d.codes_off, cb) || !inside(d.scales_off, sb) || !inside(d.g_off, 4ull * d.n_groups)) return false;
  if (d.n_groups > 1 && !inside(d.group_off_off, 4ull * (d.n_groups + 1))) return false;
  if (d.n_chan > 0 && (!inside(d.chan_off, 4ull * d.n_chan) ||
                       !inside(d.resid_off, 2ull * d.n_chan * static_cast<uint64_t>(d.rows))))
    return false;
  return true;
}

// kTrain: a trainer input is compared (x_train given); without one the lane
// loads the codes and scales of four passes at a time instead of two (the
// loop is latency-bound: a block's loads are only 9 bytes per lane).
template <bool kTrain>
__global__ void __launch_bounds__(kThreads, kTrain ? 3 : 4) replay_kernel(ReplayArgs a) {
  constexpr int kU = kTrain ? 2 : 4;                        // passes whose loads are in flight at once
  extern __shared__ int32_t smem[];
  __shared__ trace_qrecord_header h;
  __shared__ int ok;
  static_assert(sizeof(trace_qrecord_header) % 4 == 0, "header is copied as 32-bit words");
  for (int i = threadIdx.x; i < static_cast<int>(sizeof(h) / 4); i += blockDim.x)
    reinterpret_cast<uint32_t*>(&h)[i] = reinterpret_cast<const uint32_t*>(a.record)[i];
  __syncthreads();
  if (threadIdx.x == 0) {
    ok = record_ok(a, h) ? 1 : 0;
    if (blockIdx.x == 0) *a.status = ok ? QUADS_OK : QUADS_ERR_BAD_RECORD;
  }
  __syncthreads();
  if (!ok) return;
  const trace_qtensor_desc d = h.t[a.which];
  const int n = d.n_groups;
  const int64_t K = d.K;
  const int nkb = static_cast<int>(K / 16);
  const int npass = (nkb + 31) / 32;
  int32_t* off_s = smem;                                   // n + 1
  float* g_s = reinterpret_cast<float*>(smem + n + 1);     // n
  int32_t* pass_slot = smem + 2 * n + 1;                   // npass + 1
  int32_t* chan_s = pass_slot + npass + 1;                 // n_chan
  const float* g_rec = reinterpret_cast<const float*>(a.record + d.g_off);
  const int32_t* goff_rec = reinterpret_cast<const int32_t*>(a.record + d.group_off_off);
  const int32_t* chan_rec = reinterpret_cast<const int32_t*>(a.record + d.chan_off);
  const uint16_t* resid_rec = reinterpret_cast<const uint16_t*>(a.record + d.resid_off);
  for (int i = threadIdx.x; i <= n; i += blockDim.x) {
    off_s[i] = (n > 1) ? goff_rec[i] : 0;
    if (i < n) g_s[i] = g_rec[i];
  }
  if (d.n_chan) {
    for (int j = threadIdx.x; j < d.n_chan; j += blockDim.x) chan_s[j] = chan_rec[j];
    __syncthreads();
    for (int p = threadIdx.x; p <= npass; p += blockDim.x) {
      int cnt = 0;
      for (int j = 0; j < d.n_chan; ++j) {
        const int c = chan_s[j];
        cnt += (c >= 0 && c < K && c < 512 * p) ? 1 : 0;
      }
      pass_slot[p] = cnt;
    }
  }
  __syncthreads();
  RowGroups grp{n > 1 ? off_s : nullptr, n, FastDiv{1u, 1u, 0u}};
  const uint8_t* codes = a.record + d.codes_off;
  const uint8_t* scales = a.record + d.scales_off;
  const bool tiled = d.scale_layout == QUADS_SCALES_TILED;
  const int64_t ncol_tiles = ceil_div(nkb, 4);
  // rows past the last group's end hold no data (expert-ordered padding capacity)
  const int64_t rows = (n > 1) ? min(d.rows, static_cast<int64_t>(off_s[n])) : d.rows;
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  unsigned long long code_mis = 0, scale_mis = 0;
  // the codes, scales (and trainer input) of passes [p0, p0 + kU) of a row
  auto load_passes = [&](int64_t row, int p0, uint2 (&cw)[kU], uint32_t (&sc)[kU], uint32_t (&xw)[kTrain ? kU : 1][8]) {
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int kb = (p0 + u) * 32 + lane;
      if (kb < nkb) {
        cw[u] = *reinterpret_cast<const uint2*>(codes + row * (K / 2) + kb * 8);
        sc[u] = scales[tiled ? tiled_scale_offset(row, kb, ncol_tiles) : row * nkb + kb];
        if constexpr (kTrain) load_bf16x16(a.x_train + row * K + kb * 16, xw[u]);
      }
    }
  };
  // x_hat of those passes (and the mismatch counts)
  auto replay_passes = [&](int64_t row, int p0, float g, const QConsts& qc, const uint2 (&cw)[kU],
                           const uint32_t (&sc)[kU], const uint32_t (&xw)[kTrain ? kU : 1][8]) {
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int p = p0 + u;
      if (p >= npass) break;                         // warp-uniform
      const int kb = p * 32 + lane;
      QCore q{0u, 0u, 0u, 0.0f};
      uint32_t o[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
      if (kb < nkb) {
        q.lo = cw[u].x;
        q.hi = cw[u].y;
        q.scale = sc[u];
        q.sv = e4m3_value(sc[u]);
        deq_block_bf16(q, g, 1, o);
        if constexpr (kTrain) {
          const QCore t = quant_core(xw[u], qc);
          // nibbles that differ: OR-fold each nibble onto its low bit, count
          uint32_t d0 = t.lo ^ q.lo, d1 = t.hi ^ q.hi;
          d0 = (d0 | (d0 >> 1) | (d0 >> 2) | (d0 >> 3)) & 0x11111111u;
          d1 = (d1 | (d1 >> 1) | (d1 >> 2) | (d1 >> 3)) & 0x11111111u;
          code_mis += __popc(d0) + __popc(d1);
          scale_mis += (t.scale != q.scale) ? 1u : 0u;
        }
      }
      if (kb < nkb) {
        uint4* dst = reinterpret_cast<uint4*>(a.x_hat + row * K + kb * 16);
        dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
        dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
      }
      if (d.n_chan) {
        // compensation channels of this pass, rewritten after the block stores above
        replay_channel_pass(q, g, p, pass_slot[p], pass_slot[p + 1], chan_s, resid_rec + row * d.n_chan,
                            a.x_hat + row * K);
      }
    }
  };
  const int64_t first = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (!kTrain && npass <= kU) {
    // a whole row per batch: the next row's codes and scales are loaded
    // while this row is replayed
    uint2 cw[kU], ncw[kU];
    uint32_t sc[kU], nsc[kU], xw[kTrain ? kU : 1][8];
    if (first < rows) load_passes(first, 0, cw, sc, xw);
    for (int64_t row = first; row < rows; row += warps) {
      if (row + warps < rows) load_passes(row + warps, 0, ncw, nsc, xw);
      const float g = g_s[grp.of(row)];
      replay_passes(row, 0, g, make_qconsts(g), cw, sc, xw);
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        cw[u] = ncw[u];
        sc[u] = nsc[u];
      }
    }
  } else {
    for (int64_t row = first; row < rows; row += warps) {
      const float g = g_s[grp.of(row)];
      const QConsts qc = make_qconsts(g);
      for (int p0 = 0; p0 < npass; p0 += kU) {
        uint2 cw[kU];
        uint32_t sc[kU], xw[kTrain ? kU : 1][8];
        load_passes(row, p0, cw, sc, xw);
        replay_passes(row, p0, g, qc, cw, sc, xw);
      }
    }
  }
  if constexpr (kTrain) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      code_mis += __shfl_xor_sync(0xffffffffu, code_mis, o);
      scale_mis += __shfl_xor_sync(0xffffffffu, scale_mis, o);
    }
    if ((threadIdx.x & 31) == 0) {
      if (code_mis) atomicAdd(&a.counts[0], code_mis);
      if (scale_mis) atomicAdd(&a.counts[1], scale_mis);
    }
  }
}

}  // namespace
}  // namespace quads

using namespace quads;

extern "C" {

size_t trace_qrecord_layout(int layer_id, int64_t T, int k, const trace_qtensor_src* tensors, int n_tensors,
                            trace_qrecord_header* hdr) {
  if (!hdr || T < 0 || k < 0 || k > 8 || n_tensors < 0 || n_tensors > TRACE_MAX_TENSORS) return 0;
  if (n_tensors > 0 && !tensors) return 0;
  std::memset(hdr, 0, sizeof(*hdr));
  hdr->magic = TRACE_QRECORD_MAGIC;
  hdr->version = TRACE_QRECORD_VERSION;
  hdr->layer_id = layer_id;
  hdr->k = k;
  hdr->T = T;
  uint64_t off = align256(sizeof(trace_qrecord_header));
  for (int i = 0; i < n_tensors; ++i) {
    const trace_qtensor_src& s = tensors[i];
    trace_qtensor_desc& d = hdr->t[i];
    if (!s.present) continue;
    if (s.rows < 0 || s.K <= 0 || s.K % 16 || s.K > 65536 || s.n_groups < 1 || s.n_groups > 1024 ||
        s.n_chan < 0 || s.n_chan > 256 ||
        (s.scale_layout != QUADS_SCALES_LINEAR && s.scale_layout != QUADS_SCALES_TILED))
      return 0;
    d.rows = s.rows; d.K = s.K; d.n_groups = s.n_groups; d.n_chan = s.n_chan;
    d.scale_layout = s.scale_layout; d.present = 1;
    d.codes_bytes = static_cast<uint64_t>(s.rows) * (s.K / 2);
    d.scales_bytes = static_cast<uint64_t>(scale_bytes(s.rows, s.K, s.scale_layout));
    d.codes_off = off; off = align256(off + d.codes_bytes);
    d.scales_off = off; off = align256(off + d.scales_bytes);
    d.g_off = off; off = align256(off + 4ull * s.n_groups);
    if (s.n_groups > 1) { d.group_off_off = off; off = align256(off + 4ull * (s.n_groups + 1)); }
    if (s.n_chan > 0) {
      d.chan_off = off; off = align256(off + 4ull * s.n_chan);
      d.resid_off = off; off = align256(off + 2ull * s.n_chan * static_cast<uint64_t>(s.rows));
    }
  }
  if (k > 0) { hdr->topk_idx_off = off; off = align256(off + 4ull * static_cast<uint64_t>(T) * k); }
  hdr->total_bytes = off;
  return static_cast<size_t>(off);
}

int trace_export_qrecord(int layer_id, int64_t T, int k, const int32_t* topk_idx, const trace_qtensor_src* tensors,
                         int n_tensors, void* record, size_t record_bytes, quads_stream_t stream) {
  clear_error();
  ExportArgs a;
  std::memset(&a, 0, sizeof(a));
  size_t need = trace_qrecord_layout(layer_id, T, k, tensors, n_tensors, &a.hdr);
  QUADS_REQUIRE(need > 0, QUADS_ERR_INVALID_ARG, "invalid record description");
  QUADS_REQUIRE(record && record_bytes >= need, QUADS_ERR_INVALID_ARG, "record buffer of %zu bytes required", need);
  QUADS_REQUIRE(aligned(record, 256), QUADS_ERR_INVALID_ARG, "record must be 256-byte aligned");
  QUADS_REQUIRE(k == 0 || topk_idx, QUADS_ERR_INVALID_ARG, "topk_idx required when k > 0");
  int n = 0;
  auto add = [&](const void* src, uint64_t off, uint64_t bytes) -> int {
    if (bytes == 0) return QUADS_OK;
    if (!src) return set_error(QUADS_ERR_INVALID_ARG, "null section pointer");
    if (src == static_cast<const uint8_t*>(record) + off) return QUADS_OK;   // produced in place
    a.seg[n].src = static_cast<const uint8_t*>(src);
    a.seg[n].dst_off = off;
    a.seg[n].bytes = bytes;
    ++n;
    return QUADS_OK;
  };
  for (int i = 0; i < n_tensors; ++i) {
    const trace_qtensor_src& s = tensors[i];
    const trace_qtensor_desc& d = a.hdr.t[i];
    if (!s.present) continue;
    QUADS_TRY(add(s.codes, d.codes_off, d.codes_bytes));
    QUADS_TRY(add(s.scales, d.scales_off, d.scales_bytes));
    QUADS_TRY(add(s.g, d.g_off, 4ull * s.n_groups));
    if (s.n_groups > 1) QUADS_TRY(add(s.group_off, d.group_off_off, 4ull * (s.n_groups + 1)));
    if (s.n_chan > 0) {
      QUADS_TRY(add(s.chan, d.chan_off, 4ull * s.n_chan));
      QUADS_TRY(add(s.resid, d.resid_off, 2ull * s.n_chan * static_cast<uint64_t>(s.rows)));
    }
  }
  if (k > 0) QUADS_TRY(add(topk_idx, a.hdr.topk_idx_off, 4ull * static_cast<uint64_t>(T) * k));
  a.n_seg = n;
  uint64_t biggest = 16;
  for (int i = 0; i < n; ++i) biggest = a.seg[i].bytes > biggest ? a.seg[i].bytes : biggest;
  int64_t bx = ceil_div(static_cast<int64_t>(biggest / 16), kThreads);
  int64_t cap = num_sms() * 4;
  dim3 grid(static_cast<unsigned>(bx < 1 ? 1 : (bx > cap ? cap : bx)), static_cast<unsigned>(n > 0 ? n : 1));
  export_kernel<<<grid, kThreads, 0, stream>>>(a, static_cast<uint8_t*>(record));
  count_launches(1);
  return check_launch("export_kernel");
}

int trace_replay_qrecord(const void* record, size_t record_bytes, int layer_id, int which, int64_t rows, int64_t K,
                         const uint16_t* x_train, uint16_t* x_hat, unsigned long long* counts, int32_t* status,
                         quads_stream_t stream) {
  clear_error();
  QUADS_REQUIRE(record && x_hat && status, QUADS_ERR_INVALID_ARG, "record, x_hat and status must be non-null");
  QUADS_REQUIRE(record_bytes >= sizeof(trace_qrecord_header), QUADS_ERR_BAD_RECORD, "record too small");
  QUADS_REQUIRE(aligned(record, 256), QUADS_ERR_INVALID_ARG, "record must be 256-byte aligned");
  QUADS_REQUIRE(which >= 0 && which < TRACE_MAX_TENSORS, QUADS_ERR_INVALID_ARG, "which must be 0 or 1");
  QUADS_REQUIRE(rows >= 0 && K > 0 && K % 16 == 0 && K <= 65536, QUADS_ERR_UNSUPPORTED_SHAPE,
                "K must be a positive multiple of 16 up to 65536");
  QUADS_REQUIRE(aligned(x_hat, 16) && (!x_train || aligned(x_train, 16)), QUADS_ERR_INVALID_ARG,
                "x_hat and x_train must be 16-byte aligned");
  QUADS_REQUIRE(!x_train || counts, QUADS_ERR_INVALID_ARG, "counts required with x_train");
  QUADS_REQUIRE(rows * (K / 16) < (int64_t(1) << 31), QUADS_ERR_UNSUPPORTED_SHAPE, "tensor above 2^31 blocks");
  ReplayArgs a{static_cast<const uint8_t*>(record), record_bytes, layer_id, which, rows, K, x_train, x_hat, counts,
               status, make_fastdiv(static_cast<uint32_t>(K / 16))};
  // worst case: group offsets and scales of 1024 groups, the pass table and 256 channels
  size_t smem = (2 * 1024 + 1) * 4 + (static_cast<size_t>((K / 16 + 31) / 32) + 1 + 256) * 4;
  auto kernel = x_train ? replay_kernel<true> : replay_kernel<false>;
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
    return set_error(QUADS_ERR_CUDA, "cannot raise shared memory of replay_kernel");
  const int grid = persistent_grid(reinterpret_cast<const void*>(kernel), kThreads, smem, ceil_div(rows, 8));
  kernel<<<grid, kThreads, smem, stream>>>(a);
  count_launches(1);
  return check_launch("replay_kernel");
}

}  // extern "C"
