// NVFP4 grouped expert GEMM with QUADS residual compensation, for sm_100a.
//
// Method: the rollout runs its MoE expert GEMMs as native NVFP4 W4A4
// ([QUADS-fr §1]); on the high-residual input channels a correction term is
// computed and added to the quantized output, so that the W4A4 GEMM still
// does the bulk of the work ([QUADS-fr §2.2.B], [QUADS-es §2.2.B]):
//   Y = g_a g_w (A_fp4 (x) W_fp4) + R_C . Wc
//
// Design (one persistent CTA per SM, 320 threads, warp-specialized):
//   warp 0 lane 0  TMA producer: 128x256 FP4 tiles of A and W (128-byte
//                  swizzle) and their 512-byte block-scale tiles (bulk copy)
//                  into a multi-stage shared-memory ring; per output tile the
//                  BF16 compensation operands R [128 x |C|] and Wc [128 x |C|]
//                  (32-byte swizzle, 16 channels per box).
//   warps 6..9     one per TMEM lane quarter: load each stage's block scales
//                  from shared memory and write them into a TMEM slot with
//                  tcgen05.st (two per warp and stage), then signal the MMA
//                  thread.  A tcgen05.cp per 512-byte tile would cost the
//                  issuing thread more than the MMAs that read the scales.
//   warp 1         allocates 512 TMEM columns; lane 0 issues
//                  tcgen05.mma kind::mxf4nvf4 (block16
//                  E4M3 scales, K = 64 per instruction) into a double-buffered
//                  FP32 accumulator, then tcgen05.mma kind::f16 (BF16) for
//                  R_C . Wc into a second accumulator.
//   warps 2..5     epilogue: tcgen05.ld both accumulators, y = G * acc + comp,
//                  BF16 rows staged in shared memory (64-byte swizzle),
//                  TMA tensor stores of 32 x 32 boxes.
// TMEM columns: [0,128) and [128,256) main accumulators, [256,384) the
// compensation accumulator, [384,512) four slots of scale factors.
// Tiles are (expert, 128-row block, 128-column block); experts' row segments
// are 128-aligned by the permutation, so no tile straddles two experts.
// No TMA multicast is used anywhere.
//
// Every wait on an mbarrier is bounded (a global-timer limit); on expiry the
// kernel records a timeout in a device status word, lets in-flight copies and
// MMAs finish (bounded again), frees its TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"

namespace quads {

__device__ unsigned int g_wait_status = 0u;

unsigned int* wait_status_word() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_wait_status) != cudaSuccess) return nullptr;
  return static_cast<unsigned int*>(p);
}

namespace {

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int kStageRowBytes = 128;                 // 256 FP4 elements per row per stage
constexpr int kMmaKBytes = 32;                      // 64 FP4 elements per MMA
constexpr int kABytes = BM * kStageRowBytes;        // 16384
constexpr int kBBytes = BN * kStageRowBytes;        // 16384
constexpr int kSfBytes = 4 * 512;                   // scales of 4 MMAs for 128 rows
constexpr int kStageBytes = kABytes + kBBytes + 2 * kSfBytes;   // 36864
constexpr int kCompChunkBytes = 128 * 32;           // 128 rows x 16 BF16
// W4A16 stage (K = 64) for bn weight rows per tile: BF16 activations
// (128 x 64), the weights dequantized to BF16 by the converter warps
// (bn x 64), the weights' FP4 codes (bn x 32 bytes), their 512-byte scale
// tiles (one per 128 rows), padded to 1024 bytes
constexpr int kW16ABytes = BM * 128;
__host__ __device__ constexpr int w16_codes_off(int bn) { return kW16ABytes + bn * 128; }
__host__ __device__ constexpr int w16_scales_off(int bn) { return kW16ABytes + bn * 160; }
__host__ __device__ constexpr int stage_bytes(bool w4a16, int bn) {
  return w4a16 ? w16_scales_off(bn) + 1024 : kStageBytes;          // 37888 (bn 128), 58368 (bn 256)
}
constexpr int kOutChunkBytes = 32 * 64;             // 32 rows x 32 BF16 output columns
constexpr int kOutStageBytes = 4 * 2 * kOutChunkBytes;   // 4 epilogue warps, 2 buffers each
constexpr int kThreads = 320;                    // 10 warps
// The quantizing epilogue does twice the work per column, so its kernel has
// two epilogue warps per TMEM lane quarter (warps 2-5 and 10-13), each taking
// every other 32-column chunk.
__host__ __device__ constexpr int epi_warps(bool quant) { return quant ? 8 : 4; }
// The W4A16 kernel's weight conversion is on its critical path, so it has
// eight converter warps (6-13), one weight row per thread for 256-row tiles.
__host__ __device__ constexpr int conv_warps(bool w4a16) { return w4a16 ? 8 : 0; }
__host__ __device__ constexpr int threads_for(bool quant, bool w4a16 = false) {
  return (quant || w4a16) ? 448 : kThreads;
}
__host__ __device__ constexpr int out_stage_bytes(bool quant) { return epi_warps(quant) * 2 * kOutChunkBytes; }
constexpr int kSfSlots = 4;                      // scale-factor buffers in TMEM
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kCompCol = 256;
constexpr uint32_t kSfCol = 384;
constexpr int kMaxStages = 8;
constexpr int kMaxChan = 128;
constexpr uint64_t kGemmTimeoutNs = 4000000000ull;
constexpr uint64_t kDrainTimeoutNs = 500000000ull;

// Instruction descriptors (tcgen05 "instruction descriptor" format):
// kind::mxf4nvf4: A/B format E2M1 (1) at bits 7-9 / 10-12, K-major, N>>3 at
// bit 17, scale format UE4M3 (0) at bit 23, M>>4 at bit 24, dense K = 64.
constexpr uint32_t kIdescFp4 = (1u << 7) | (1u << 10) | (uint32_t(BN >> 3) << 17) | (uint32_t(BM >> 4) << 24);
// kind::f16: D format F32 (1) at bits 4-5, A/B BF16 (1), K-major, N>>3, M>>4.
__host__ __device__ constexpr uint32_t idesc_bf16(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(n >> 3) << 17) | (uint32_t(BM >> 4) << 24);
}
constexpr uint32_t kIdescBf16 = idesc_bf16(BN);

struct GemmParams {
  const uint8_t* a_scales;
  const uint8_t* w_scales;
  const float* g_a;
  const float* g_w;
  const int32_t* expert_off;
  uint16_t* y;
  unsigned int* amax_bits;   // SwiGLU epilogue: per-expert max |h| (float bits), or null
  // SwiGLU epilogue with NVFP4 quantization of h (per-expert scale from amax_h_in)
  const float* amax_h_in;    // [E]
  const int32_t* chan_h;     // [n_chan_h]: h's compensation channels
  uint8_t* h_codes;          // [rows_cap][F/2]
  uint8_t* h_scales;         // tiled over rows_cap x F
  uint16_t* h_resid;         // [rows_cap][n_chan_h]
  float* g_h_out;            // [E]
  int n_chan_h;
  // FP4 compensation: NVFP4 residual / weight-column operands appended to the
  // reduction axis (nkb_comp 64-wide K blocks; tiled scales)
  const uint8_t* a2_scales;  // [rows_cap] x Kc
  const uint8_t* w2_scales;  // [E * N] x Kc
  int nkb_comp;
  int g_a_per_expert;
  int E;
  int rows_cap;              // rows of a_codes, y and the h outputs
  int N;
  int K;
  int n_chan;
  int comp_cw;               // channels per box of the correction operands (wide and decode tiles)
  int stages;
  uint64_t timeout_ns;
};

// ------------------------------------------------------------ PTX wrappers

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t global_timer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
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

// Bounded wait for the phase with the given parity.  Returns false if the
// limit expired (recording a timeout and raising the CTA's abort flag) or if
// another role already aborted.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          uint64_t limit_ns) {
  if (mbar_test(bar, parity)) return true;
  const uint64_t t0 = global_timer();
  while (true) {
    if (mbar_test(bar, parity)) return true;
    if (abort_flag != nullptr && *abort_flag) return false;
    if (global_timer() - t0 > limit_ns) {
      if (abort_flag != nullptr) *abort_flag = 1;
      atomicOr(&g_wait_status, 1u);
      return false;
    }
  }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int x, int y, int z, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

// Store a box of the output from shared memory through TMA (bulk-group
// completion tracked by the issuing thread).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y), "r"(src)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void st_shared_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t ld_shared_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
// 16 consecutive TMEM columns of this warp's 32 lanes from registers.
__device__ __forceinline__ void tmem_store16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void mma_fp4(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}
__device__ __forceinline__ void mma_bf16(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}
// kind::f16 with A read from tensor memory (a: its TMEM address, K-major
// rows on the lanes, two 16-bit elements per 32-bit column)
__device__ __forceinline__ void mma_bf16_tmem_a(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc,
                                                uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
      "r"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void tmem_load32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_load16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptors (tcgen05 format: start >> 4 at bit 0,
// leading-byte offset >> 4 at bit 16, stride-byte offset >> 4 at bit 32,
// version 1 at bit 46, swizzle mode at bit 61).
__device__ __forceinline__ uint64_t desc_kmajor_sw128(uint32_t addr) {
  return uint64_t((addr >> 4) & 0x3FFFu) | (uint64_t(1) << 16) | (uint64_t(1024 >> 4) << 32) | (uint64_t(1) << 46) |
         (uint64_t(2) << 61);
}
__device__ __forceinline__ uint64_t desc_kmajor_sw32(uint32_t addr) {
  return uint64_t((addr >> 4) & 0x3FFFu) | (uint64_t(1) << 16) | (uint64_t(256 >> 4) << 32) | (uint64_t(1) << 46) |
         (uint64_t(6) << 61);
}

// K-major descriptor for rows of row_bytes = 32, 64 or 128 bytes stored with
// the swizzle of that width (8-row groups of 8 * row_bytes).
__device__ __forceinline__ uint64_t desc_kmajor_rows(uint32_t addr, int row_bytes) {
  const uint64_t layout = row_bytes == 128 ? 2u : (row_bytes == 64 ? 4u : 6u);
  return uint64_t((addr >> 4) & 0x3FFFu) | (uint64_t(1) << 16) | (uint64_t((8 * row_bytes) >> 4) << 32) |
         (uint64_t(1) << 46) | (layout << 61);
}

// out_s[0] = 0, out_s[e + 1] = out_s[e] + ceil(max(off_s[e + 1] - off_s[e], 0) / rows) * mult
// for e < E <= 256; run by one whole warp (each lane a run of experts, a
// shuffle scan across lanes).
__device__ __forceinline__ void warp_block_prefix(int32_t* out_s, const int32_t* off_s, int E, int rows, int mult,
                                                  int lane) {
  const int per = (E + 31) / 32, e0 = lane * per;
  int sum = 0;
  for (int i = 0; i < per; ++i)
    if (e0 + i < E) sum += (max(off_s[e0 + i + 1] - off_s[e0 + i], 0) + rows - 1) / rows * mult;
  int incl = sum;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += v;
  }
  int run = incl - sum;
  if (lane == 0) out_s[0] = 0;
  for (int i = 0; i < per; ++i)
    if (e0 + i < E) {
      run += (max(off_s[e0 + i + 1] - off_s[e0 + i], 0) + rows - 1) / rows * mult;
      out_s[e0 + i + 1] = run;
    }
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

__device__ __forceinline__ int expert_of_row(const int32_t* off_s, int E, int row) {
  int lo = 0, hi = E - 1;                 // last expert whose segment starts at or before row
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (off_s[mid] <= row) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// ------------------------------------------------------------------ kernel

// One output before rounding: fp32(G * acc + comp) in one FMA, or
// fp32(G * acc) without compensation.
__device__ __forceinline__ float epi_value(uint32_t acc, float G, bool has_comp, uint32_t comp) {
  return has_comp ? __fmaf_rn(__uint_as_float(acc), G, __uint_as_float(comp)) : __fmul_rn(__uint_as_float(acc), G);
}

// kSwiglu: the W rows of every 128-row tile are 64 gate rows then the 64
// matching up rows; the epilogue writes h = silu(y_gate) * y_up (64 columns
// per tile) instead of y, and the per-expert max |h|.
// NVFP4 quantization of one lane's 32 consecutive h values (one row, h
// columns [col0, col0 + 32), two blocks of 16) with decode scale g: codes,
// the two tiled scales, and the residual of every compensation channel in
// the chunk; the lane holding a row's first chunk also zeroes its padding
// channel slots.  Same operations as quads_quantize_nvfp4 (quant_core).
__device__ __forceinline__ void quantize_h_chunk(const GemmParams& p, const uint32_t (&o)[16], float g,
                                                 const int32_t* chanh_s, const int32_t* hslot_s, int row, int col0,
                                                 bool first_chunk) {
  const int Fh = p.N / 2;
  const QConsts qc = make_qconsts(g);
  uint32_t w0[8], w1[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    w0[i] = o[i];
    w1[i] = o[8 + i];
  }
  const QCore q0 = quant_core(w0, qc), q1 = quant_core(w1, qc);
  const int64_t r = row;
  *reinterpret_cast<uint4*>(p.h_codes + r * (Fh / 2) + col0 / 2) = make_uint4(q0.lo, q0.hi, q1.lo, q1.hi);
  // blocks col0 / 16 and the next: adjacent bytes of one tiled scale row (col0 / 16 is even)
  const int64_t so = tiled_scale_offset(r, col0 / 16, Fh / 64);
  *reinterpret_cast<uint16_t*>(p.h_scales + so) = static_cast<uint16_t>(q0.scale | (q1.scale << 8));
  if (p.n_chan_h) {
    const int slo = hslot_s[col0 / 32], shi = hslot_s[col0 / 32 + 1];
    for (int j = slo; j < shi; ++j) {
      const int cc = chanh_s[j] - col0, b = cc >> 4, bit = cc & 15;
      uint32_t word = 0;
#pragma unroll
      for (int i = 0; i < 16; ++i) word = (i == (cc >> 1)) ? o[i] : word;
      const float hv = bf16_bits_to_float((cc & 1) ? (word >> 16) : (word & 0xFFFFu));
      const uint32_t lo = b ? q1.lo : q0.lo, hi = b ? q1.hi : q0.hi;
      const uint32_t code = (((bit < 8) ? lo : hi) >> (4 * (bit & 7))) & 15u;
      const float dq = deq_f32(code, b ? q1.sv : q0.sv, g);
      p.h_resid[r * p.n_chan_h + j] = static_cast<uint16_t>(float_to_bf16_bits(__fsub_rn(hv, dq)));
    }
    if (first_chunk)
      for (int j = hslot_s[Fh / 32]; j < p.n_chan_h; ++j) p.h_resid[r * p.n_chan_h + j] = 0;
  }
}

// kQuant (with kSwiglu): h is also NVFP4-quantized in the epilogue with the
// per-expert scale g_e = fp32(amax_h_in[e] / 2688): codes, tiled scales and
// the residual channels, exactly as quads_quantize_nvfp4 of h with that
// amax; h itself is stored only when y is non-null.
//
// kW4A16: the trainer-side GEMM Y = X . W_fq^T with BF16 activations X and
// the weights given as NVFP4 codes and scales: warps 6-9 turn each stage's
// FP4 weight tile into W_fq = bf16(fp32(val(q) val(s)) g_w[e]) in shared
// memory (the 128-byte-swizzled K-major layout the MMA reads), and the MMA
// is kind::f16 (BF16 x BF16, FP32 accumulate); the epilogue stores fp32 acc.
template <bool kSwiglu, bool kQuant, bool kW4A16, int kBN = BN>
__global__ void __launch_bounds__(threads_for(kQuant, kW4A16), 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                        const __grid_constant__ CUtensorMap tm_r, const __grid_constant__ CUtensorMap tm_wc,
                        const __grid_constant__ CUtensorMap tm_y, const __grid_constant__ CUtensorMap tm_a2,
                        const __grid_constant__ CUtensorMap tm_b2, GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const base_ptr = smem_raw + (base - raw);
  const int S = p.stages;
  const int nch = p.n_chan / 16;
  constexpr int kSB = stage_bytes(kW4A16, kBN);
  static_assert(kBN == BN || kW4A16, "256-row weight tiles are the W4A16 kernel's only");
  const uint32_t comp_r = base + S * kSB;
  const uint32_t comp_wc = comp_r + nch * kCompChunkBytes;
  const uint32_t out_stage = comp_wc + nch * kCompChunkBytes;     // 1024-byte aligned
  constexpr int kEpi = epi_warps(kQuant);
  const uint32_t bar0 = out_stage + out_stage_bytes(kQuant);        // 8-byte aligned
  // barrier addresses
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (S + s); };
  const uint32_t comp_full = bar0 + 8u * (2 * S);
  const uint32_t comp_empty = comp_full + 8;
  const uint32_t acc_full0 = comp_full + 16;       // two barriers
  const uint32_t acc_empty0 = comp_full + 32;      // two barriers
  const uint32_t compacc_empty = comp_full + 48;
  const uint32_t drain_bar = comp_full + 56;
  auto sf_full = [&](int i) { return comp_full + 64 + 8u * i; };            // kSfSlots barriers
  auto sf_empty = [&](int i) { return comp_full + 64 + 8u * (kSfSlots + i); };
  auto conv_bar = [&](int s) { return comp_full + 64 + 8u * (2 * kSfSlots + s); };   // W4A16: S barriers
  uint8_t* const misc = base_ptr + (comp_full + 64 + 8u * (2 * kSfSlots + S) + 8 - base);
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(misc);
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  int32_t* const off_s = reinterpret_cast<int32_t*>(misc + 16);
  float* const gscale_s = reinterpret_cast<float*>(off_s + p.E + 1);   // g_a(e) * g_w[e]
  // kQuant: h's per-expert scale, its channels, and per 32-column chunk of h
  // the first channel slot at or after the chunk (valid channels ascend)
  float* const gh_s = gscale_s + p.E;                                  // E
  int32_t* const chanh_s = reinterpret_cast<int32_t*>(gh_s + p.E);     // n_chan_h
  int32_t* const hslot_s = chanh_s + p.n_chan_h;                       // N / 64 + 1

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(comp_full, 1);
    mbar_init(comp_empty, 1);
    mbar_init(acc_full0, 1);
    mbar_init(acc_full0 + 8, 1);
    mbar_init(acc_empty0, kEpi);              // one arrival per epilogue warp
    mbar_init(acc_empty0 + 8, kEpi);
    mbar_init(compacc_empty, kEpi);
    mbar_init(drain_bar, 1);
    for (int i = 0; i < kSfSlots; ++i) {
      mbar_init(sf_full(i), 4);                 // one arrival per scale warp
      mbar_init(sf_empty(i), 1);
    }
    for (int s = 0; s < S; ++s) mbar_init(conv_bar(s), conv_warps(true));   // one arrival per converter warp
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  for (int i = threadIdx.x; i <= p.E; i += blockDim.x) {
    off_s[i] = p.expert_off[i];
    if (i < p.E) gscale_s[i] = kW4A16 ? p.g_w[i] : __fmul_rn(p.g_a[p.g_a_per_expert ? i : 0], p.g_w[i]);
  }
  if constexpr (kQuant) {
    const int Fh = p.N / 2;
    for (int i = threadIdx.x; i < p.E; i += blockDim.x) {
      gh_s[i] = __fdiv_rn(p.amax_h_in[i], kNvfp4Range);
      if (blockIdx.x == 0 && p.g_h_out != nullptr) p.g_h_out[i] = gh_s[i];
    }
    for (int j = threadIdx.x; j < p.n_chan_h; j += blockDim.x) chanh_s[j] = p.chan_h[j];
    __syncthreads();
    for (int qc = threadIdx.x; qc <= Fh / 32; qc += blockDim.x) {
      int cnt = 0;
      for (int j = 0; j < p.n_chan_h; ++j) cnt += (chanh_s[j] >= 0 && chanh_s[j] < Fh && chanh_s[j] < 32 * qc) ? 1 : 0;
      hslot_s[qc] = cnt;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int n_ntiles = p.N / kBN;
  // row tiles below expert_off[E], never past the buffers' rows_cap rows
  const int total = (min(off_s[p.E], p.rows_cap) / BM) * n_ntiles;
  const int nkb_total = p.K / 64;                 // MMAs along K
  const int nks_main = kW4A16 ? nkb_total : (nkb_total + 3) / 4;   // pipeline stages along K
  const int nks = nks_main + (p.nkb_comp + 3) / 4; // then the FP4 compensation's stages
  const int n_col_tiles = nkb_total;              // 512-byte scale tiles per 128-row band

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer
    int it = 0;
    uint32_t cph = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
      const int mt = t / n_ntiles, nt = t - mt * n_ntiles;
      const int m0 = mt * BM;
      const int e = expert_of_row(off_s, p.E, m0);
      const int brow = e * p.N + nt * kBN;
      for (int ks = 0; ks < nks; ++ks, ++it) {
        const int s = it % S;
        const uint32_t ph = (it / S) & 1;
        if (!mbar_wait(empty_bar(s), ph ^ 1u, abort_flag, p.timeout_ns)) { ok = false; break; }
        const uint32_t st = base + s * kSB;
        if constexpr (kW4A16) {
          // BF16 activations (64 per row), FP4 weight codes, their scale tile
          mbar_expect_tx(full_bar(s), kW16ABytes + kBN * 32 + (kBN / 128) * 512);
          tma_load_2d(st, &tm_a, ks * 64, m0, full_bar(s));
          tma_load_2d(st + w16_codes_off(kBN), &tm_b, ks * kMmaKBytes, brow, full_bar(s));
#pragma unroll
          for (int b = 0; b < kBN / 128; ++b)
            bulk_load(st + w16_scales_off(kBN) + b * 512,
                      p.w_scales + (static_cast<int64_t>(brow / BM + b) * n_col_tiles + ks) * 512, 512, full_bar(s));
        } else if (ks < nks_main) {
          const int nkb = min(4, nkb_total - ks * 4);
          mbar_expect_tx(full_bar(s), kABytes + kBBytes + 2 * nkb * 512);
          tma_load_2d(st, &tm_a, ks * kStageRowBytes, m0, full_bar(s));
          tma_load_2d(st + kABytes, &tm_b, ks * kStageRowBytes, brow, full_bar(s));
          bulk_load(st + kABytes + kBBytes, p.a_scales + (static_cast<int64_t>(mt) * n_col_tiles + ks * 4) * 512,
                    nkb * 512, full_bar(s));
          bulk_load(st + kABytes + kBBytes + kSfBytes,
                    p.w_scales + (static_cast<int64_t>(brow / BM) * n_col_tiles + ks * 4) * 512, nkb * 512,
                    full_bar(s));
        } else {
          // FP4 compensation: one 128 x 32-byte box (32-byte swizzle) per K block
          const int j0 = (ks - nks_main) * 4;
          const int nkb = min(4, p.nkb_comp - j0);
          mbar_expect_tx(full_bar(s), 2 * nkb * (kCompChunkBytes + 512));
          for (int j = 0; j < nkb; ++j) {
            tma_load_2d(st + j * kCompChunkBytes, &tm_a2, (j0 + j) * kMmaKBytes, m0, full_bar(s));
            tma_load_2d(st + kABytes + j * kCompChunkBytes, &tm_b2, (j0 + j) * kMmaKBytes, brow, full_bar(s));
          }
          bulk_load(st + kABytes + kBBytes, p.a2_scales + (static_cast<int64_t>(mt) * p.nkb_comp + j0) * 512,
                    nkb * 512, full_bar(s));
          bulk_load(st + kABytes + kBBytes + kSfBytes,
                    p.w2_scales + (static_cast<int64_t>(brow / BM) * p.nkb_comp + j0) * 512, nkb * 512,
                    full_bar(s));
        }
      }
      if (ok && nch) {
        if (!mbar_wait(comp_empty, cph ^ 1u, abort_flag, p.timeout_ns)) { ok = false; break; }
        mbar_expect_tx(comp_full, 2 * nch * kCompChunkBytes);
        for (int j = 0; j < nch; ++j) {
          tma_load_2d(comp_r + j * kCompChunkBytes, &tm_r, j * 16, m0, comp_full);
          tma_load_2d(comp_wc + j * kCompChunkBytes, &tm_wc, j * 16, brow, comp_full);
        }
        cph ^= 1u;
      }
    }
    if (!ok) {
      // let every copy this thread issued land before the CTA can exit
      for (int i = (it > S ? it - S : 0); i < it; ++i)
        mbar_wait(full_bar(i % S), (i / S) & 1, nullptr, kDrainTimeoutNs);
      if (nch) mbar_wait(comp_full, cph ^ 1u, nullptr, kDrainTimeoutNs);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------------- MMA
    int it = 0, tc = 0;
    uint32_t cph = 0, caph = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++tc) {
      const int buf = tc & 1;
      const uint32_t aph = (tc >> 1) & 1;
      if (!mbar_wait(acc_empty0 + 8 * buf, aph ^ 1u, abort_flag, p.timeout_ns)) { ok = false; break; }
      tc_fence_after();
      const uint32_t dacc = tmem + buf * kBN;
      for (int ks = 0; ks < nks; ++ks, ++it) {
        const int s = it % S;
        const uint32_t ph = (it / S) & 1;
        const int slot = it % kSfSlots;
        if (!mbar_wait(full_bar(s), ph, abort_flag, p.timeout_ns)) { ok = false; break; }
        if constexpr (kW4A16) {
          if (!mbar_wait(conv_bar(s), ph, abort_flag, p.timeout_ns)) { ok = false; break; }
          tc_fence_after();
          const uint32_t st = base + s * kSB;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)      // four K = 16 BF16 MMAs per stage
            mma_bf16(dacc, desc_kmajor_sw128(st + kk * 32), desc_kmajor_sw128(st + kW16ABytes + kk * 32),
                     idesc_bf16(kBN), (ks | kk) != 0 ? 1u : 0u);
          tc_commit(empty_bar(s));
          continue;
        }
        if (!mbar_wait(sf_full(slot), (it / kSfSlots) & 1, abort_flag, p.timeout_ns)) { ok = false; break; }
        tc_fence_after();
        const uint32_t st = base + s * kSB;
        const uint32_t tsfa = tmem + kSfCol + slot * 32;
        const uint32_t tsfb = tsfa + 16;
        if (ks < nks_main) {
          const int nkb = min(4, nkb_total - ks * 4);
          for (int kb = 0; kb < nkb; ++kb)
            mma_fp4(dacc, desc_kmajor_sw128(st + kb * kMmaKBytes), desc_kmajor_sw128(st + kABytes + kb * kMmaKBytes),
                    kIdescFp4, tsfa + kb * 4, tsfb + kb * 4, (ks | kb) != 0 ? 1u : 0u);
        } else {
          const int nkb = min(4, p.nkb_comp - (ks - nks_main) * 4);
          for (int kb = 0; kb < nkb; ++kb)
            mma_fp4(dacc, desc_kmajor_sw32(st + kb * kCompChunkBytes),
                    desc_kmajor_sw32(st + kABytes + kb * kCompChunkBytes), kIdescFp4, tsfa + kb * 4, tsfb + kb * 4,
                    1u);
        }
        tc_commit(empty_bar(s));
        tc_commit(sf_empty(slot));
      }
      if (!ok) break;
      if (nch) {
        if (!mbar_wait(comp_full, cph, abort_flag, p.timeout_ns)) { ok = false; break; }
        tc_fence_after();
        cph ^= 1u;
        if (!mbar_wait(compacc_empty, caph ^ 1u, abort_flag, p.timeout_ns)) { ok = false; break; }
        tc_fence_after();
        caph ^= 1u;
        for (int j = 0; j < nch; ++j)
          mma_bf16(tmem + kCompCol, desc_kmajor_sw32(comp_r + j * kCompChunkBytes),
                   desc_kmajor_sw32(comp_wc + j * kCompChunkBytes), kIdescBf16, j != 0 ? 1u : 0u);
        tc_commit(comp_empty);
      }
      tc_commit(acc_full0 + 8 * buf);
    }
    if (!ok) {
      // wait for every MMA and scale copy already issued before TMEM is freed
      tc_commit(drain_bar);
      mbar_wait(drain_bar, 0, nullptr, kDrainTimeoutNs);
    }
  } else if (kW4A16 && warp >= 6) {
    // ------------------------------------------- W4A16 weight converters
    // Thread r of warps 6..13 owns weight row r of the tile (threads past
    // the tile's rows idle): the row's 64 FP4 codes (32 bytes) and 4 block
    // scales (in the 512-byte tile of its 128-row band) become 64 BF16 values
    // of W_fq written as that row of the 128-byte-swizzled K-major tile
    // (16-byte chunk j at j ^ (row % 8)), the layout a TMA load with 128-byte
    // swizzle produces.
    const int r0 = (warp - 6) * 32 + lane;                            // 0..255
    int it = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
      const int m0 = (t / n_ntiles) * BM;
      const float g = gscale_s[expert_of_row(off_s, p.E, m0)];
      for (int ks = 0; ks < nks; ++ks, ++it) {
        const int s = it % S;
        const bool w_ok = mbar_wait(full_bar(s), (it / S) & 1, abort_flag, p.timeout_ns);
        if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
        const uint32_t st = base + s * kSB;
#pragma unroll
        for (int h = 0; h < (kBN + 255) / 256; ++h) {
          const int r = r0 + 256 * h;
          if (r >= kBN) break;
          const uint32_t cw = st + w16_codes_off(kBN) + r * 32;
          const uint4 c0 = ld_shared_v4(cw), c1 = ld_shared_v4(cw + 16);
          const uint4 sv = ld_shared_v4(st + w16_scales_off(kBN) + (r >> 7) * 512 + (r & 31) * 16);
          const int qr = (r >> 5) & 3;
          const uint32_t sc = qr == 0 ? sv.x : (qr == 1 ? sv.y : (qr == 2 ? sv.z : sv.w));
          const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
          const uint32_t row = st + kW16ABytes + r * 128;
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const QCore q{words[2 * b], words[2 * b + 1], (sc >> (8 * b)) & 0xFFu, 0.0f};
            uint32_t o[8];
            deq_block_bf16(q, g, 1, o);
            st_shared_v4(row + (static_cast<uint32_t>((2 * b) ^ (r & 7)) << 4), o[0], o[1], o[2], o[3]);
            st_shared_v4(row + (static_cast<uint32_t>((2 * b + 1) ^ (r & 7)) << 4), o[4], o[5], o[6], o[7]);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(conv_bar(s));
      }
    }
  } else if (warp >= 6 && warp <= 9) {
    // ------------------------------------------------------- block scales
    // Warps 6..9, one per TMEM lane quarter q: lane i of the quarter reads
    // row i (16 bytes: rows i, i + 32, i + 64, i + 96 x 4 scales) of each of
    // the stage's 512-byte scale tiles and writes them to the slot's columns
    // (4 per 64-wide K block), the layout the block-scaled MMA reads for all
    // 128 rows.  Two tcgen05.st per warp and stage.
    int it = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
      for (int ks = 0; ks < nks; ++ks, ++it) {
        const int s = it % S, slot = it % kSfSlots;
        bool w_ok = mbar_wait(full_bar(s), (it / S) & 1, abort_flag, p.timeout_ns);
        if (w_ok) w_ok = mbar_wait(sf_empty(slot), ((it / kSfSlots) & 1) ^ 1u, abort_flag, p.timeout_ns);
        if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sf = base + s * kSB + kABytes + kBBytes + lane * 16;
        const uint32_t tsf = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16) + kSfCol + slot * 32;
        uint32_t ra[16], rb[16];
#pragma unroll
        for (int kb = 0; kb < 4; ++kb) {        // tiles past the stage's last K block are never read
          const uint4 a = ld_shared_v4(sf + kb * 512);
          const uint4 b = ld_shared_v4(sf + kSfBytes + kb * 512);
          ra[4 * kb] = a.x; ra[4 * kb + 1] = a.y; ra[4 * kb + 2] = a.z; ra[4 * kb + 3] = a.w;
          rb[4 * kb] = b.x; rb[4 * kb + 1] = b.y; rb[4 * kb + 2] = b.z; rb[4 * kb + 3] = b.w;
        }
        tmem_store16(tsf, ra);
        tmem_store16(tsf + 16, rb);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(sf_full(slot));
      }
    }
  } else if ((warp >= 2 && warp <= 5) || (kQuant && warp >= 10)) {
    // ----------------------------------------------------------- epilogue
    // Each warp owns 32 accumulator rows (its TMEM lane quarter).  Per
    // 32-column chunk: TMEM -> registers -> y = G * acc + comp -> BF16 row in
    // a 2 KB shared buffer -> one TMA store of the 32 x 32 box.  Two buffers
    // per warp; a buffer is rewritten only after its previous store has read it.
    // With two warps per quarter, warp 10 + i takes the odd chunks of warp 2 + i.
    const int q = warp & 3;
    const int ew = warp <= 5 ? warp - 2 : warp - 6;                   // 0..kEpi-1
    constexpr int kStride = kEpi / 4;
    const int c0 = warp >= 10 ? 1 : 0;
    const uint32_t stg = out_stage + ew * 2 * kOutChunkBytes;
    int tc = 0, nstore = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++tc) {
      const int mt = t / n_ntiles, nt = t - mt * n_ntiles;
      const int m0 = mt * BM;
      const int e = expert_of_row(off_s, p.E, m0);
      const int buf = tc & 1;
      const uint32_t ph = (tc >> 1) & 1;
      if (!mbar_wait(acc_full0 + 8 * buf, ph, abort_flag, p.timeout_ns)) break;
      tc_fence_after();
      const float G = kW4A16 ? 1.0f : gscale_s[e];      // W4A16: g_w is inside W_fq
      const uint32_t lane_base = tmem + (static_cast<uint32_t>(q * 32) << 16);
      constexpr int kChunks = kSwiglu ? kBN / 64 : kBN / 32;   // 32 output columns each
#pragma unroll 1
      for (int c = c0; c < kChunks; c += kStride, ++nstore) {
        const bool last = c + kStride >= kChunks;         // this warp's last TMEM read of the tile
        uint32_t o[16];
        unsigned int hmax = 0u;
        if constexpr (!kSwiglu) {
          uint32_t v[32], w[32];
          tmem_load32(lane_base + buf * kBN + c * 32, v);
          if (nch) tmem_load32(lane_base + kCompCol + c * 32, w);
          tmem_wait_ld();
          if (last) {
            // every TMEM read of this tile is done: hand the accumulators back
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
              mbar_arrive(acc_empty0 + 8 * buf);
              if (nch) mbar_arrive(compacc_empty);
            }
          }
#pragma unroll
          for (int j = 0; j < 16; ++j)
            o[j] = pack_bf16x2(epi_value(v[2 * j], G, nch, w[2 * j]),
                               epi_value(v[2 * j + 1], G, nch, w[2 * j + 1]));
        } else {
          // gate columns [32c, 32c + 32) and the matching up columns 64 further,
          // read 16 at a time to keep the register footprint small
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            // gate columns of 128-column half c / 2; the up columns follow 64 later
            const uint32_t col = (c >> 1) * 128 + (c & 1) * 32 + hf * 16;
            uint32_t vg[16], vu[16], wg[16], wu[16];
            tmem_load16(lane_base + buf * kBN + col, vg);
            tmem_load16(lane_base + buf * kBN + 64 + col, vu);
            if (nch) {
              tmem_load16(lane_base + kCompCol + col, wg);
              tmem_load16(lane_base + kCompCol + 64 + col, wu);
            }
            tmem_wait_ld();
            if (last && hf == 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) {
                mbar_arrive(acc_empty0 + 8 * buf);
                if (nch) mbar_arrive(compacc_empty);
              }
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              // y rounded to BF16 exactly as the plain epilogue stores it, then
              // SwiGLU in FP32 as quads_swiglu computes it from that y
              const uint32_t yg = pack_bf16x2(epi_value(vg[2 * j], G, nch, wg[2 * j]),
                                              epi_value(vg[2 * j + 1], G, nch, wg[2 * j + 1]));
              const uint32_t yu = pack_bf16x2(epi_value(vu[2 * j], G, nch, wu[2 * j]),
                                              epi_value(vu[2 * j + 1], G, nch, wu[2 * j + 1]));
              float r[2];
#pragma unroll
              for (int hl = 0; hl < 2; ++hl) {
                const float gt = bf16_bits_to_float(hl ? (yg >> 16) : (yg & 0xFFFFu));
                const float ut = bf16_bits_to_float(hl ? (yu >> 16) : (yu & 0xFFFFu));
                r[hl] = __fmul_rn(__fdividef(gt, 1.0f + __expf(-gt)), ut);
              }
              o[hf * 8 + j] = pack_bf16x2(r[0], r[1]);
              hmax = max(hmax, max(o[hf * 8 + j] & 0x7FFFu, (o[hf * 8 + j] >> 16) & 0x7FFFu));
            }
          }
        }
        if constexpr (kQuant) quantize_h_chunk(p, o, gh_s[e], chanh_s, hslot_s, m0 + q * 32 + lane,
                                               nt * (kBN / 2) + c * 32, nt == 0 && c == 0);
        if (!kQuant || p.y != nullptr) {
          const uint32_t sb = stg + (nstore & 1) * kOutChunkBytes;
          if (lane == 0) bulk_wait_read_1();
          __syncwarp();
          // 64-byte swizzle (the store's tensor map): 16-byte chunk j of row r sits
          // at chunk j ^ ((r >> 1) & 3), so the 32 lanes' row stores hit all banks
          const uint32_t row_addr = sb + lane * 64;
          const uint32_t sw = (lane >> 1) & 3u;
#pragma unroll
          for (int j = 0; j < 4; ++j)
            st_shared_v4(row_addr + ((j ^ sw) << 4), o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tm_y, sb, (kSwiglu ? nt * (kBN / 2) : nt * kBN) + c * 32, m0 + q * 32);
            bulk_commit();
          }
        }
        if constexpr (kSwiglu) {
          hmax = __reduce_max_sync(0xffffffffu, hmax);
          if (lane == 0 && hmax != 0u && p.amax_bits != nullptr) atomicMax(&p.amax_bits[e], hmax << 16);
        }
      }
    }
    if (lane == 0) bulk_wait_all();
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------------------
// Pair tiles: two CTAs on two SMs compute one 256-row x 256-column tile with
// tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 64 per instruction).
//
// Why: the single-CTA kernel above is bound by how fast TMA fills each SM's
// shared memory (about 30 bytes per clock per SM), not by its MMAs.  In a
// pair, CTA r holds rows [128 r, 128 r + 128) of A and rows
// [128 r, 128 r + 128) of the tile's 256 weight rows; the MMA issued by CTA 0
// reads both CTAs' halves, so every SM loads 8 KB per 128 x 256 x 64 product
// instead of 8 KB per 128 x 128 x 64: half the bytes per FLOP.  Each CTA
// loads only its own halves (no multicast).
//
// Roles (448 threads, 14 warps, the same in both CTAs):
//   warp 0 lane 0  TMA producer into this CTA's stage ring: its A rows, its
//                  weight rows, the block scales of its A rows and of all 256
//                  weight rows; then the BF16 correction operands R and Wc
//                  (16-channel chunks) as extra stages after the K loop.
//   warps 2..5     one per TMEM lane quarter: write each stage's block scales
//                  into a TMEM slot of this CTA (tcgen05.st), or for the
//                  correction stages rescale R in place to R / G; then
//                  arrive on CTA 0's barrier of that slot.
//   warp 1         allocates 512 TMEM columns in both CTAs (cta_group::2);
//                  in CTA 0 lane 0 issues the MMAs once both CTAs' slots are
//                  ready and commits their completion to both CTAs' barriers.
//   warps 6..13    epilogue, two warps per lane quarter (128 accumulator
//                  columns each): y = G * acc, BF16, TMA stores; or SwiGLU
//                  (and the NVFP4 quantization of h) as the single-CTA kernel.
// TMEM per CTA: [0, 256) the accumulator (one buffer), [256, 512) four
// scale-factor slots of 64 columns (A scales in 16, B scales in 32).
//
// The BF16 correction is accumulated into the FP4 accumulator: the MMA adds
// (R / G) . Wc, so y = G * acc = G * A.W + R . Wc up to the rounding of
// R / G, computed as bf16(fp32(R * fp32(1 / G))) (a relative 2^-9 + 2^-23 of
// each correction term).  G = g_a g_w[e] of the
// tile's expert; a zero G (an all-zero input or expert) gives R / G = 0.
//
// Rows: each expert's 128-aligned segment is cut into 256-row pair blocks
// from its first row; a segment with an odd number of 128-row blocks ends in
// a pair block whose second half belongs to the next expert: CTA 1 loads no
// A rows for it and its results are not stored.
constexpr int PBM = 256;
constexpr int PBN = 256;
constexpr int kPairHalfBytes = 128 * kStageRowBytes;               // 16384: 128 rows x 256 FP4
constexpr int kPairSfaBytes = 4 * 512;                              // its 128 A rows, 4 MMAs
constexpr int kPairSfbBytes = 2 * 4 * 512;                          // all 256 weight rows, 4 MMAs
// this CTA's weight rows per stage: half of the 256 in a pair, all 256 alone
__host__ __device__ constexpr int wide_b_bytes(bool pair) { return pair ? kPairHalfBytes : 2 * kPairHalfBytes; }
__host__ __device__ constexpr int wide_stage_bytes(bool pair) {
  return kPairHalfBytes + wide_b_bytes(pair) + kPairSfaBytes + kPairSfbBytes;       // 38912 or 55296
}
constexpr int kPairThreads = 448;
constexpr int kPairSfSlots = 4;
constexpr uint32_t kPairSfCol = 256;
constexpr uint32_t kPairSlotCols = 64;
constexpr int kPairEpiWarps = 8;
// instruction descriptors with M = 256 (the pair's rows), N = 256
constexpr uint32_t kIdescFp4Pair = (1u << 7) | (1u << 10) | (uint32_t(PBN >> 3) << 17) | (uint32_t(PBM >> 4) << 24);
constexpr uint32_t kIdescBf16Pair =
    (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(PBN >> 3) << 17) | (uint32_t(PBM >> 4) << 24);
// one CTA alone: M = 128, N = 256
constexpr uint32_t kIdescFp4Wide = (1u << 7) | (1u << 10) | (uint32_t(PBN >> 3) << 17) | (uint32_t(128 >> 4) << 24);
constexpr uint32_t kIdescBf16Wide =
    (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(PBN >> 3) << 17) | (uint32_t(128 >> 4) << 24);
// output staging: each epilogue warp stages 32 rows x 64 columns at a time
__host__ __device__ constexpr int pair_out_bytes() { return kPairEpiWarps * 2 * kOutChunkBytes; }

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}
// Address of the same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ bool mbar_test_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait (as mbar_wait) on a barrier that the peer CTA also arrives on.
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                                  uint64_t limit_ns) {
  if (mbar_test_cluster(bar, parity)) return true;
  const uint64_t t0 = global_timer();
  while (true) {
    if (mbar_test_cluster(bar, parity)) return true;
    if (abort_flag != nullptr && *abort_flag) return false;
    if (global_timer() - t0 > limit_ns) {
      if (abort_flag != nullptr) *abort_flag = 1;
      atomicOr(&g_wait_status, 1u);
      return false;
    }
  }
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// Completion of this thread's earlier MMAs arrives on the barrier at the same
// offset in every CTA of `mask`.
__device__ __forceinline__ void tc_commit_pair_mc(uint32_t bar, uint16_t mask) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::
                   "r"(bar), "h"(mask)
               : "memory");
}
__device__ __forceinline__ void tc_commit_pair(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mma_fp4_pair(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa,
                                             uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}
__device__ __forceinline__ void mma_bf16_pair(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

// h = silu(gate) * up for two packed BF16 pairs, in FP32 as quads_swiglu
// computes it, rounded to a packed BF16 pair.
__device__ __forceinline__ uint32_t swiglu_bf16x2(uint32_t yg, uint32_t yu) {
  float r[2];
#pragma unroll
  for (int hl = 0; hl < 2; ++hl) {
    const float gt = bf16_bits_to_float(hl ? (yg >> 16) : (yg & 0xFFFFu));
    const float ut = bf16_bits_to_float(hl ? (yu >> 16) : (yu & 0xFFFFu));
    r[hl] = __fmul_rn(__fdividef(gt, 1.0f + __expf(-gt)), ut);
  }
  return pack_bf16x2(r[0], r[1]);
}

// Stage 32 rows x 32 BF16 columns (this lane's row: 16 packed words) in a
// 2 KB buffer with the store map's 64-byte swizzle.
__device__ __forceinline__ void stage_chunk(uint32_t sb, int lane, const uint32_t (&o)[16]) {
  const uint32_t row_addr = sb + lane * 64;
  const uint32_t sw = (lane >> 1) & 3u;
#pragma unroll
  for (int j = 0; j < 4; ++j) st_shared_v4(row_addr + ((j ^ sw) << 4), o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
}

template <bool kSwiglu, bool kQuant, bool kPair>
__global__ void __launch_bounds__(kPairThreads, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                             const __grid_constant__ CUtensorMap tm_r, const __grid_constant__ CUtensorMap tm_wc,
                             const __grid_constant__ CUtensorMap tm_y, GemmParams p) {
  static_assert(kSwiglu || !kQuant, "the quantizing epilogue follows SwiGLU");
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const base_ptr = smem_raw + (base - raw);
  const int S = p.stages;
  constexpr int kSB = wide_stage_bytes(kPair);
  constexpr int kBB = wide_b_bytes(kPair);
  constexpr int kRows = kPair ? PBM : 128;        // rows of a tile
  // BF16 correction operands in boxes of cw channels (rows of 2 cw bytes, the
  // swizzle of that width), 64 channels per stage: R [128 x cw] and this
  // CTA's Wc rows [128 or 256 x cw] per box
  const int cw = p.comp_cw, cps = 64 / cw;
  const int rcb = 128 * 2 * cw, wcb = (kPair ? 128 : 256) * 2 * cw;
  const uint32_t rank = kPair ? cluster_ctarank() : 0u;
  const uint32_t out_stage = base + S * kSB;
  constexpr int kOutB = pair_out_bytes();
  const uint32_t bar0 = out_stage + kOutB;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (S + s); };
  auto sf_full = [&](int i) { return bar0 + 8u * (2 * S + i); };
  auto sf_empty = [&](int i) { return bar0 + 8u * (2 * S + kPairSfSlots + i); };
  const uint32_t acc_full = bar0 + 8u * (2 * S + 2 * kPairSfSlots);
  const uint32_t acc_empty = acc_full + 8;
  const uint32_t drain_bar = acc_full + 16;
  uint8_t* const misc = base_ptr + (drain_bar + 8 - base);
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(misc);
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  int32_t* const off_s = reinterpret_cast<int32_t*>(misc + 16);       // E + 1, clamped to rows_cap
  int32_t* const pb_s = off_s + p.E + 1;                                 // E + 1: first pair block of each expert
  float* const gscale_s = reinterpret_cast<float*>(pb_s + p.E + 1);     // g_a(e) * g_w[e]
  float* const gh_s = gscale_s + p.E;                                    // kQuant: h's per-expert scale
  int32_t* const chanh_s = reinterpret_cast<int32_t*>(gh_s + p.E);     // n_chan_h
  int32_t* const hslot_s = chanh_s + p.n_chan_h;                        // N / 64 + 1

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    prefetch_tensormap(&tm_a);
    prefetch_tensormap(&tm_b);
    if (p.n_chan) {
      prefetch_tensormap(&tm_r);
      prefetch_tensormap(&tm_wc);
    }
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int i = 0; i < kPairSfSlots; ++i) {
      mbar_init(sf_full(i), kPair ? 2 * 4 : 4);   // four scale warps in each CTA
      mbar_init(sf_empty(i), 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, kPair ? 2 * kPairEpiWarps : kPairEpiWarps);   // every epilogue warp of both CTAs
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    if constexpr (kPair) {
      tmem_alloc_pair(smem_addr(tmem_slot), kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_addr(tmem_slot), kTmemCols);
      tmem_relinquish();
    }
  }
  for (int i = threadIdx.x; i <= p.E; i += blockDim.x) {
    off_s[i] = min(p.expert_off[i], p.rows_cap);
    if (i < p.E) gscale_s[i] = __fmul_rn(p.g_a[p.g_a_per_expert ? i : 0], p.g_w[i]);
  }
  if constexpr (kQuant) {
    const int Fh = p.N / 2;
    for (int i = threadIdx.x; i < p.E; i += blockDim.x) {
      gh_s[i] = __fdiv_rn(p.amax_h_in[i], kNvfp4Range);
      if (blockIdx.x == 0 && p.g_h_out != nullptr) p.g_h_out[i] = gh_s[i];
    }
    for (int j = threadIdx.x; j < p.n_chan_h; j += blockDim.x) chanh_s[j] = p.chan_h[j];
    __syncthreads();
    for (int qc = threadIdx.x; qc <= Fh / 32; qc += blockDim.x) {
      int cnt = 0;
      for (int j = 0; j < p.n_chan_h; ++j) cnt += (chanh_s[j] >= 0 && chanh_s[j] < Fh && chanh_s[j] < 32 * qc) ? 1 : 0;
      hslot_s[qc] = cnt;
    }
  }
  __syncthreads();
  if (warp == 2) warp_block_prefix(pb_s, off_s, p.E, kRows, 1, lane);
  tc_fence_before();
  if constexpr (kPair)
    cluster_sync_all();                // barriers initialized and TMEM allocated in both CTAs
  else
    __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int n_ntiles = p.N / PBN;
  const int total = pb_s[p.E] * n_ntiles;
  const int nkb_total = p.K / 64;
  const int nks_main = (nkb_total + 3) / 4;
  const int nch = p.n_chan / cw;                  // cw-channel boxes of the BF16 correction
  const int nks = nks_main + (nch + cps - 1) / cps;
  const int n_col_tiles = nkb_total;
  const int cluster_id = kPair ? blockIdx.x >> 1 : blockIdx.x, n_clusters = kPair ? gridDim.x >> 1 : gridDim.x;
  // pair tile t: expert e, first row m0, column tile nt, and whether its
  // second 128 rows belong to e
  auto tile_of = [&](int t, int& e, int& m0, int& nt, bool& hi_valid) {
    const int pb = t / n_ntiles;
    nt = t - pb * n_ntiles;
    e = expert_of_row(pb_s, p.E, pb);
    m0 = off_s[e] + kRows * (pb - pb_s[e]);
    hi_valid = !kPair || m0 + 128 < off_s[e + 1];
  };

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer
    int it = 0;
    bool ok = true;
    for (int t = cluster_id; t < total && ok; t += n_clusters) {
      int e, m0, nt;
      bool hi_valid;
      tile_of(t, e, m0, nt, hi_valid);
      const bool av = rank == 0 || hi_valid;      // this CTA's A rows belong to the tile's expert
      const int row0 = m0 + 128 * static_cast<int>(rank);
      const int brow = e * p.N + nt * PBN;        // the tile's first weight row
      const int myb = brow + 128 * static_cast<int>(rank);
      for (int ks = 0; ks < nks; ++ks, ++it) {
        const int s = it % S;
        const uint32_t ph = (it / S) & 1;
        if (!mbar_wait_cluster(empty_bar(s), ph ^ 1u, abort_flag, p.timeout_ns)) { ok = false; break; }
        const uint32_t st = base + s * kSB;
        if (ks < nks_main) {
          const int nkb = min(4, nkb_total - ks * 4);
          mbar_expect_tx(full_bar(s), kBB + 2 * nkb * 512 + (av ? kPairHalfBytes + nkb * 512 : 0));
          if (av) {
            tma_load_2d(st, &tm_a, ks * kStageRowBytes, row0, full_bar(s));
            bulk_load(st + kPairHalfBytes + kBB,
                      p.a_scales + (static_cast<int64_t>(row0 / 128) * n_col_tiles + ks * 4) * 512, nkb * 512,
                      full_bar(s));
          }
          tma_load_2d(st + kPairHalfBytes, &tm_b, ks * kStageRowBytes, myb, full_bar(s));   // 128 or 256 rows
#pragma unroll
          for (int b = 0; b < 2; ++b)
            bulk_load(st + kPairHalfBytes + kBB + kPairSfaBytes + b * 2048,
                      p.w_scales + (static_cast<int64_t>(brow / 128 + b) * n_col_tiles + ks * 4) * 512, nkb * 512,
                      full_bar(s));
        } else {
          const int j0 = (ks - nks_main) * cps, nj = min(cps, nch - j0);
          mbar_expect_tx(full_bar(s), nj * (wcb + (av ? rcb : 0)));
          for (int j = 0; j < nj; ++j) {
            if (av) tma_load_2d(st + j * rcb, &tm_r, (j0 + j) * cw, row0, full_bar(s));
            tma_load_2d(st + kPairHalfBytes + j * wcb, &tm_wc, (j0 + j) * cw, myb, full_bar(s));
          }
        }
      }
    }
    if (!ok) {
      for (int i = (it > S ? it - S : 0); i < it; ++i) mbar_wait(full_bar(i % S), (i / S) & 1, nullptr, kDrainTimeoutNs);
    }
  } else if (warp == 1 && lane == 0 && rank == 0) {
    // ------------------------------------------------- MMA (CTA 0 of the pair)
    int it = 0, tc = 0;
    int s = 0, slot = 0;                          // stage and scale slot of `it`
    uint32_t ph = 0, sph = 0;                     // their phases
    bool ok = true;
    for (int t = cluster_id; t < total && ok; t += n_clusters, ++tc) {
      if (!mbar_wait_cluster(acc_empty, (tc & 1) ^ 1u, abort_flag, p.timeout_ns)) { ok = false; break; }
      tc_fence_after();
      for (int ks = 0; ks < nks; ++ks, ++it) {
        // One CTA: a scale slot per stage, and the scale warps' arrival (made
        // after they saw the stage's data land) is the only wait.  Pair: the
        // slots cycle on their own and the stage's own barrier is waited too.
        // (the cluster-scope acquire is used even for a CTA alone: its
        // waits measured faster at tile boundaries)
        if (!mbar_wait_cluster(sf_full(slot), sph, abort_flag, p.timeout_ns)) { ok = false; break; }
        if (kPair && !mbar_wait(full_bar(s), ph, abort_flag, p.timeout_ns)) { ok = false; break; }
        tc_fence_after();
        const uint32_t st = base + s * kSB;
        const uint32_t tsfa = tmem + kPairSfCol + slot * kPairSlotCols;
        const uint32_t tsfb = tsfa + 16;
        if (ks < nks_main) {
          const int nkb = min(4, nkb_total - ks * 4);
          for (int kb = 0; kb < nkb; ++kb) {
            const uint64_t da = desc_kmajor_sw128(st + kb * kMmaKBytes);
            const uint64_t db = desc_kmajor_sw128(st + kPairHalfBytes + kb * kMmaKBytes);
            const uint32_t acc = (ks | kb) != 0 ? 1u : 0u;
            if constexpr (kPair)
              mma_fp4_pair(tmem, da, db, kIdescFp4Pair, tsfa + 4 * kb, tsfb + 8 * kb, acc);
            else
              mma_fp4(tmem, da, db, kIdescFp4Wide, tsfa + 4 * kb, tsfb + 8 * kb, acc);
          }
        } else {
          const int nj = min(cps, nch - (ks - nks_main) * cps);
          for (int j = 0; j < nj; ++j)
            for (int kk = 0; kk < cw / 16; ++kk) {      // K = 16 channels per MMA, 32 bytes along the row
              const uint64_t da = desc_kmajor_rows(st + j * rcb + kk * 32, 2 * cw);
              const uint64_t db = desc_kmajor_rows(st + kPairHalfBytes + j * wcb + kk * 32, 2 * cw);
              if constexpr (kPair)
                mma_bf16_pair(tmem, da, db, kIdescBf16Pair, 1u);
              else
                mma_bf16(tmem, da, db, kIdescBf16Wide, 1u);
            }
        }
        if constexpr (kPair) {
          tc_commit_pair_mc(empty_bar(s), 3);
          tc_commit_pair_mc(sf_empty(slot), 3);
        } else {
          tc_commit(empty_bar(s));           // frees the stage and its scale slot
        }
        if (++s == S) { s = 0; ph ^= 1u; }
        if constexpr (kPair) {
          if (++slot == kPairSfSlots) { slot = 0; sph ^= 1u; }
        } else {
          slot = s;
          sph = ph;
        }
      }
      if (!ok) break;
      if constexpr (kPair)
        tc_commit_pair_mc(acc_full, 3);
      else
        tc_commit(acc_full);
    }
    if (!ok) {
      if constexpr (kPair)
        tc_commit_pair(drain_bar);
      else
        tc_commit(drain_bar);
      mbar_wait(drain_bar, 0, nullptr, kDrainTimeoutNs);
    }
  } else if (warp >= 2 && warp <= 5) {
    // ------------------------------------- block scales / rescaled residuals
    // Lane i of the warp for lane quarter q writes TMEM lane 32 q + i of the
    // slot: A scales of rows i + 32 j in column 4 kb + j and weight scales of
    // rows i + 32 j (j < 8) in column 16 + 8 kb + j, for MMA kb of the stage
    // (the layout a tcgen05.cp .32x128b.warpx4 of each 512-byte tile gives).
    const int q = warp & 3;
    int it = 0;
    bool ok = true;
    for (int t = cluster_id; t < total && ok; t += n_clusters) {
      int e, m0, nt;
      bool hi_valid;
      tile_of(t, e, m0, nt, hi_valid);
      const bool av = rank == 0 || hi_valid;
      const float G = gscale_s[e];
      const float Ginv = G > 0.0f ? __frcp_rn(G) : 0.0f;     // R / G as R * fp32(1 / G)
      for (int ks = 0; ks < nks; ++ks, ++it) {
        // one CTA: the stage's data landing implies its slot is free (the
        // producer refilled the stage only after the MMAs that read it)
        const int s = it % S, slot = kPair ? it % kPairSfSlots : s;
        bool w_ok = mbar_wait(full_bar(s), (it / S) & 1, abort_flag, p.timeout_ns);
        if (kPair && w_ok)
          w_ok = mbar_wait_cluster(sf_empty(slot), ((it / kPairSfSlots) & 1) ^ 1u, abort_flag, p.timeout_ns);
        if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
        tc_fence_after();
        const uint32_t st = base + s * kSB;
        if (ks < nks_main) {
          const uint32_t sfa = st + kPairHalfBytes + kBB + lane * 16;
          const uint32_t sfb = sfa + kPairSfaBytes;
          const uint32_t tsf = tmem + (static_cast<uint32_t>(q * 32) << 16) + kPairSfCol + slot * kPairSlotCols;
          uint32_t ra[16], rb[16], rc[16];
#pragma unroll
          for (int kb = 0; kb < 4; ++kb) {       // tiles past the stage's last K block are never read
            const uint4 a = ld_shared_v4(sfa + kb * 512);
            const uint4 b0 = ld_shared_v4(sfb + kb * 512);
            const uint4 b1 = ld_shared_v4(sfb + 2048 + kb * 512);
            ra[4 * kb] = a.x; ra[4 * kb + 1] = a.y; ra[4 * kb + 2] = a.z; ra[4 * kb + 3] = a.w;
            uint32_t* d = kb < 2 ? rb : rc;
            const int o = (kb & 1) * 8;
            d[o] = b0.x; d[o + 1] = b0.y; d[o + 2] = b0.z; d[o + 3] = b0.w;
            d[o + 4] = b1.x; d[o + 5] = b1.y; d[o + 6] = b1.z; d[o + 7] = b1.w;
          }
          tmem_store16(tsf, ra);
          tmem_store16(tsf + 16, rb);
          tmem_store16(tsf + 32, rc);
          tmem_wait_st();
          tc_fence_before();
        } else if (av) {
          // R / G rounded to BF16 (as R * fp32(1 / G)), in place: this lane's row of each box
          // (2 cw bytes; the swizzle permutes 16-byte pieces within the row)
          // (each lane starts at another 16-byte piece: the rows of a
          // quarter warp then fall in distinct banks)
          const int nj = min(cps, nch - (ks - nks_main) * cps);
          const int units = cw / 8, rot = (q * 32 + lane) >> (cw == 64 ? 0 : (cw == 32 ? 1 : 2));
          for (int j = 0; j < nj; ++j) {
            const uint32_t ad = st + j * rcb + (q * 32 + lane) * 2 * cw;
            for (int hh = 0; hh < units; ++hh) {
              const int h = (hh + rot) & (units - 1);
              const uint4 v = ld_shared_v4(ad + 16 * h);
              uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float lo = __fmul_rn(bf16_bits_to_float(w[i] & 0xFFFFu), Ginv);
                const float hi = __fmul_rn(bf16_bits_to_float(w[i] >> 16), Ginv);
                w[i] = pack_bf16x2(lo, hi);
              }
              st_shared_v4(ad + 16 * h, w[0], w[1], w[2], w[3]);
            }
          }
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) {
          if constexpr (kPair)
            mbar_arrive_cluster(mapa_shared(sf_full(slot), 0));
          else
            mbar_arrive(sf_full(slot));
        }
      }
    }
  } else if (warp >= 6) {
    // ----------------------------------------------------------- epilogue
    // Warp 6 + 4 hs + i reads TMEM lane quarter q = warp % 4 and accumulator
    // columns [128 hs, 128 hs + 128).  Two 32-column chunks are read at a
    // time; after the last read the accumulator is handed back to the MMA,
    // and the rest of the tile's epilogue overlaps the next tile's MMAs.
    const int q = warp & 3, hs = (warp - 6) >> 2;
    const uint32_t stg = out_stage + (warp - 6) * (kOutB / kPairEpiWarps);
    const uint32_t lead_acc_empty = kPair ? mapa_shared(acc_empty, 0) : acc_empty;
    auto arrive_acc_empty = [&]() {
      if constexpr (kPair)
        mbar_arrive_cluster(lead_acc_empty);
      else
        mbar_arrive(lead_acc_empty);
    };
    int tc = 0;
    for (int t = cluster_id; t < total; t += n_clusters, ++tc) {
      int e, m0, nt;
      bool hi_valid;
      tile_of(t, e, m0, nt, hi_valid);
      const bool valid = rank == 0 || hi_valid;
      if (!mbar_wait_cluster(acc_full, tc & 1, abort_flag, p.timeout_ns)) break;
      tc_fence_after();
      const int row = m0 + 128 * static_cast<int>(rank) + q * 32 + lane;
      const float G = gscale_s[e];
      const uint32_t acc = tmem + (static_cast<uint32_t>(q * 32) << 16) + hs * 128;
      if (!valid) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) arrive_acc_empty();
        continue;
      }
      // the warp's stores of its previous tile must have read the staging buffer
      if (lane == 0) bulk_wait_read_0();
      __syncwarp();
      auto release = [&]() {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) arrive_acc_empty();
      };
      if constexpr (!kSwiglu) {
        // all 128 columns are read and rounded to BF16 before the accumulator
        // is handed back; then two halves of 64 columns go out through the
        // warp's two 2 KB buffers
        uint32_t ob[4][16];
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) {
          uint32_t v[2][32];
          tmem_load32(acc + c2 * 64, v[0]);
          tmem_load32(acc + c2 * 64 + 32, v[1]);
          tmem_wait_ld();
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int j = 0; j < 16; ++j)
              ob[2 * c2 + h][j] = pack_bf16x2(__fmul_rn(__uint_as_float(v[h][2 * j]), G),
                                              __fmul_rn(__uint_as_float(v[h][2 * j + 1]), G));
        }
        release();
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) {
          if (c2 == 1) {
            if (lane == 0) bulk_wait_read_0();      // the first half's stores have read the buffers
            __syncwarp();
          }
#pragma unroll
          for (int h = 0; h < 2; ++h) stage_chunk(stg + h * kOutChunkBytes, lane, ob[2 * c2 + h]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
#pragma unroll
            for (int h = 0; h < 2; ++h)
              tma_store_2d(&tm_y, stg + h * kOutChunkBytes, nt * PBN + hs * 128 + c2 * 64 + h * 32, row - lane);
            bulk_commit();
          }
        }
      } else {
        unsigned int hmax = 0u;
        // gate columns [32 c, 32 c + 32) of the warp's 128 and the up columns
        // 64 further, for both chunks, rounded to BF16 before the
        // accumulator is handed back; SwiGLU follows from the rounded values
        uint32_t yg[2][16], yu[2][16];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t vg[32], vu[32];
          tmem_load32(acc + c * 32, vg);
          tmem_load32(acc + 64 + c * 32, vu);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            yg[c][j] = pack_bf16x2(__fmul_rn(__uint_as_float(vg[2 * j]), G), __fmul_rn(__uint_as_float(vg[2 * j + 1]), G));
            yu[c][j] = pack_bf16x2(__fmul_rn(__uint_as_float(vu[2 * j]), G), __fmul_rn(__uint_as_float(vu[2 * j + 1]), G));
          }
        }
        release();
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t o[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            o[j] = swiglu_bf16x2(yg[c][j], yu[c][j]);
            hmax = max(hmax, max(o[j] & 0x7FFFu, (o[j] >> 16) & 0x7FFFu));
          }
          const int hcol = nt * (PBN / 2) + hs * 64 + c * 32;
          if constexpr (kQuant) quantize_h_chunk(p, o, gh_s[e], chanh_s, hslot_s, row, hcol, hcol == 0);
          if (!kQuant || p.y != nullptr) stage_chunk(stg + c * kOutChunkBytes, lane, o);
        }
        if (!kQuant || p.y != nullptr) {
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
#pragma unroll
            for (int c = 0; c < 2; ++c)
              tma_store_2d(&tm_y, stg + c * kOutChunkBytes, nt * (PBN / 2) + hs * 64 + c * 32, row - lane);
            bulk_commit();
          }
        }
        hmax = __reduce_max_sync(0xffffffffu, hmax);
        if (lane == 0 && hmax != 0u && p.amax_bits != nullptr) atomicMax(&p.amax_bits[e], hmax << 16);
      }
    }
    if (lane == 0) bulk_wait_all();
  }
  __syncwarp();
  tc_fence_before();
  if constexpr (kPair)
    cluster_sync_all();                // every MMA has completed and no peer arrival is pending
  else
    __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    if constexpr (kPair)
      tmem_dealloc_pair(tmem, kTmemCols);
    else
      tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Decode tiles: the weights as the MMA's M operand.
//
// At decode sizes an expert receives a handful of rows, so a 128-row A tile
// is mostly padding and the GEMM is a stream of the experts' weights.  Here
// the roles of the operands are swapped: D^T = W . A^T, with 128 weight rows
// on the MMA's M (TMEM lanes) and up to 128 of the expert's rows on its N
// (TMEM columns).  A work unit is (expert, 256 consecutive weight rows, a
// block of up to 128 of the expert's rows), as two M = 128 halves sharing one
// token tile (one 128-row box; rows past the expert's segment read as
// zeros or belong to the next segment and only feed accumulator columns
// that are never stored).
//
//   halves      plain: weight rows [0, 128) and [128, 256) of the unit
//               (one 256-row box).  kSwiglu: the unit covers 128 h columns;
//               half 0 holds their 128 gate rows and half 1 the 128 up rows
//               (weight rows are interleaved 64 gate / 64 up, so each half
//               is rows 0-63 or 64-127 of the unit's two 128-row blocks,
//               one 3D box), so lane i of both accumulators belongs to the
//               same h column and SwiGLU needs no exchange between lanes.
//   roles       as the one-CTA 128 x 256 kernel: warp 0 lane 0 loads, warps
//               2..5 write each stage's scales into TMEM (the weights' as the
//               A scales, the rows' as the B scales) or rescale R to R / G,
//               warp 1 lane 0 issues the MMAs, warps 6..13 the epilogue (two
//               per lane quarter, 64 accumulator columns = rows each).
//   TMEM        [0, 128) half 0, [128, 256) half 1 (one buffer, handed back
//               right after it is read); [256, 512) four scale slots of 64
//               columns: half 0 A scales at 0, half 1 at 16, B scales at 32.
//   correction  folded into the FP4 accumulator as (R / G) . Wc, R / G =
//               bf16(fp32(R * fp32(1 / G))), as the 128 x 256 kernel.
//   units       ordered expert, weight block, row block (row blocks
//               innermost, so the CTAs that share a weight block run at the
//               same time and all but one read it from L2).
constexpr int kDecRowsPerUnit = 256;                  // weight rows per unit
constexpr int kDecTok = 128;                          // expert rows per unit at most
constexpr int kDecHalfBytes = 128 * kStageRowBytes;  // 16384
constexpr int kDecXOff = 2 * kDecHalfBytes;           // token tile
constexpr int kDecWsfOff = kDecXOff + kDecTok * kStageRowBytes;   // weight scale tiles (two 128-row blocks)
constexpr int kDecXsfOff = kDecWsfOff + 2 * 4 * 512;             // token scale tile
constexpr int kDecStageBytes = kDecXsfOff + 4 * 512;              // 55296
constexpr int kDecWcOff = kDecTok * 128;                          // correction stage: Wc after R (64 channels)
constexpr int kDecBox = 128;                          // rows per TMA box of the token tile
constexpr int kDecSlots = 4;
constexpr int kDecEpiWarps = 8;
constexpr int kDecThreads = 448;

template <bool kSwiglu>
__global__ void __launch_bounds__(kDecThreads, 1)
    grouped_gemm_decode_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                               const __grid_constant__ CUtensorMap tm_r, const __grid_constant__ CUtensorMap tm_wc,
                               GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const base_ptr = smem_raw + (base - raw);
  const int S = p.stages;
  const uint32_t bar0 = base + S * kDecStageBytes;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (S + s); };
  auto sf_full = [&](int s) { return bar0 + 8u * (2 * S + s); };
  const uint32_t acc_full = bar0 + 8u * (3 * S);
  const uint32_t acc_empty = acc_full + 8;
  const uint32_t drain_bar = acc_full + 16;
  uint8_t* const misc = base_ptr + (drain_bar + 8 - base);
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(misc);
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  int32_t* const off_s = reinterpret_cast<int32_t*>(misc + 16);       // E + 1, clamped to rows_cap
  int32_t* const ub_s = off_s + p.E + 1;                                 // E + 1: first unit of each expert
  float* const gscale_s = reinterpret_cast<float*>(ub_s + p.E + 1);     // g_a(e) * g_w[e]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    prefetch_tensormap(&tm_x);
    prefetch_tensormap(&tm_w);
    if (p.n_chan) {
      prefetch_tensormap(&tm_r);
      prefetch_tensormap(&tm_wc);
    }
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
      mbar_init(sf_full(s), 4);                 // one arrival per scale warp
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, kDecEpiWarps);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  const int nwb = p.N / kDecRowsPerUnit;
  for (int i = threadIdx.x; i <= p.E; i += blockDim.x) {
    off_s[i] = min(p.expert_off[i], p.rows_cap);
    if (i < p.E) gscale_s[i] = __fmul_rn(p.g_a[p.g_a_per_expert ? i : 0], p.g_w[i]);
  }
  __syncthreads();
  if (warp == 2) warp_block_prefix(ub_s, off_s, p.E, kDecTok, nwb, lane);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int total = ub_s[p.E];
  const int nkb_total = p.K / 64;
  const int nks_main = (nkb_total + 3) / 4;
  // BF16 correction operands in boxes of cw channels (rows of 2 cw bytes, the
  // swizzle of that width), 64 channels per stage: R [128 x cw] (one box)
  // and Wc [256 x cw] (64-row boxes) per box column
  const int cw = p.comp_cw, cps = 64 / cw;
  const int rcb = kDecTok * 2 * cw, wcb = kDecRowsPerUnit * 2 * cw;
  const int nch = p.n_chan / cw;
  const int nks = nks_main + (nch + cps - 1) / cps;
  const int n_col_tiles = nkb_total;
  // unit u: expert e, its first weight row wrow (over all experts), the
  // expert-local weight block wb, the first row row0 and the number of rows
  auto unit_of = [&](int u, int& e, int& wrow, int& wb, int& row0, int& nrows) {
    e = expert_of_row(ub_s, p.E, u);
    const int ntb = (off_s[e + 1] - off_s[e] + kDecTok - 1) / kDecTok;
    const int local = u - ub_s[e];
    wb = local / ntb;
    const int tb = local - wb * ntb;
    wrow = e * p.N + wb * kDecRowsPerUnit;
    row0 = off_s[e] + kDecTok * tb;
    nrows = min(kDecTok, off_s[e + 1] - row0);
  };

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer
    int it = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
      int e, wrow, wb, row0, nrows;
      unit_of(u, e, wrow, wb, row0, nrows);
      const int nbox = (nrows + kDecBox - 1) / kDecBox;   // boxes of the token tile that hold rows
      for (int ks = 0; ks < nks; ++ks, ++it) {
        const int s = it % S;
        if (!mbar_wait(empty_bar(s), ((it / S) & 1) ^ 1u, abort_flag, p.timeout_ns)) { ok = false; break; }
        const uint32_t st = base + s * kDecStageBytes;
        if (ks < nks_main) {
          const int nkb = min(4, nkb_total - ks * 4);
          mbar_expect_tx(full_bar(s), 2 * kDecHalfBytes + 3 * nkb * 512 + nbox * kDecBox * kStageRowBytes);
          if constexpr (kSwiglu) {
            // half h: rows 64 h .. 64 h + 63 of both 128-row blocks, one 3D box
#pragma unroll
            for (int h = 0; h < 2; ++h)
              tma_load_3d(st + h * kDecHalfBytes, &tm_w, ks * kStageRowBytes, 64 * h, wrow / 128, full_bar(s));
          } else {
            tma_load_2d(st, &tm_w, ks * kStageRowBytes, wrow, full_bar(s));     // 256 rows
          }
#pragma unroll
          for (int b = 0; b < 2; ++b)
            bulk_load(st + kDecWsfOff + b * 2048,
                      p.w_scales + (static_cast<int64_t>(wrow / 128 + b) * n_col_tiles + ks * 4) * 512, nkb * 512,
                      full_bar(s));
          for (int i = 0; i < nbox; ++i)
            tma_load_2d(st + kDecXOff + i * kDecBox * kStageRowBytes, &tm_x, ks * kStageRowBytes, row0 + kDecBox * i,
                        full_bar(s));
          bulk_load(st + kDecXsfOff, p.a_scales + (static_cast<int64_t>(row0 / 128) * n_col_tiles + ks * 4) * 512,
                    nkb * 512, full_bar(s));
        } else {
          const int j0 = (ks - nks_main) * cps, nj = min(cps, nch - j0);
          mbar_expect_tx(full_bar(s), nj * (wcb + nbox * kDecBox * 2 * cw));
          for (int j = 0; j < nj; ++j) {
            const uint32_t wc = st + kDecWcOff + j * wcb;
            if constexpr (kSwiglu) {
#pragma unroll
              for (int h = 0; h < 2; ++h)
                tma_load_3d(wc + h * (wcb / 2), &tm_wc, (j0 + j) * cw, 64 * h, wrow / 128, full_bar(s));
            } else {
              tma_load_2d(wc, &tm_wc, (j0 + j) * cw, wrow, full_bar(s));
            }
            for (int i = 0; i < nbox; ++i)
              tma_load_2d(st + j * rcb + i * kDecBox * 2 * cw, &tm_r, (j0 + j) * cw, row0 + kDecBox * i, full_bar(s));
          }
        }
      }
    }
    if (!ok) {
      for (int i = (it > S ? it - S : 0); i < it; ++i) mbar_wait(full_bar(i % S), (i / S) & 1, nullptr, kDrainTimeoutNs);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------------ MMA
    int it = 0, tc = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < total && ok; u += gridDim.x, ++tc) {
      if (!mbar_wait_cluster(acc_empty, (tc & 1) ^ 1u, abort_flag, p.timeout_ns)) { ok = false; break; }
      tc_fence_after();
      for (int ks = 0; ks < nks; ++ks, ++it) {
        const int s = it % S;
        if (!mbar_wait_cluster(sf_full(s), (it / S) & 1, abort_flag, p.timeout_ns)) { ok = false; break; }
        tc_fence_after();
        const uint32_t st = base + s * kDecStageBytes;
        const uint32_t slot = tmem + kPairSfCol + s * kPairSlotCols;
        if (ks < nks_main) {
          const int nkb = min(4, nkb_total - ks * 4);
          for (int kb = 0; kb < nkb; ++kb) {
            const uint64_t dx = desc_kmajor_sw128(st + kDecXOff + kb * kMmaKBytes);
            const uint32_t acc = (ks | kb) != 0 ? 1u : 0u;
#pragma unroll
            for (int h = 0; h < 2; ++h)
              mma_fp4(tmem + 128 * h, desc_kmajor_sw128(st + h * kDecHalfBytes + kb * kMmaKBytes), dx, kIdescFp4,
                      slot + 16 * h + 4 * kb, slot + 32 + 4 * kb, acc);
          }
        } else {
          const int nj = min(cps, nch - (ks - nks_main) * cps);
          for (int j = 0; j < nj; ++j)
            for (int kk = 0; kk < cw / 16; ++kk) {      // K = 16 channels per MMA, 32 bytes along the row
              const uint64_t dr = desc_kmajor_rows(st + j * rcb + kk * 32, 2 * cw);
#pragma unroll
              for (int h = 0; h < 2; ++h)
                mma_bf16(tmem + 128 * h,
                         desc_kmajor_rows(st + kDecWcOff + j * wcb + h * (wcb / 2) + kk * 32, 2 * cw), dr,
                         kIdescBf16, 1u);
            }
        }
        tc_commit(empty_bar(s));               // frees the stage and its scale slot
      }
      if (!ok) break;
      tc_commit(acc_full);
    }
    if (!ok) {
      tc_commit(drain_bar);
      mbar_wait(drain_bar, 0, nullptr, kDrainTimeoutNs);
    }
  } else if (warp >= 2 && warp <= 5) {
    // ------------------------------------- block scales / rescaled residuals
    // Lane i of the warp for lane quarter q writes TMEM lane 32 q + i of the
    // stage's slot: for MMA kb, column 4 kb + j of each half holds the scales
    // of its A rows i + 32 j, and column 32 + 4 kb + j those of token rows
    // i + 32 j.  A SwiGLU half takes rows 0..63 (gate) or 64..127 (up) of
    // both 128-row weight blocks: words 0, 1 or 2, 3 of each block's tile.
    const int q = warp & 3;
    int it = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
      int e, wrow, wb, row0, nrows;
      unit_of(u, e, wrow, wb, row0, nrows);
      const float G = gscale_s[e];
      const float Ginv = G > 0.0f ? __frcp_rn(G) : 0.0f;     // R / G as R * fp32(1 / G)
      const bool my_row = q * 32 + lane < (nrows + kDecBox - 1) / kDecBox * kDecBox;   // a loaded token row
      for (int ks = 0; ks < nks; ++ks, ++it) {
        const int s = it % S;
        const bool w_ok = mbar_wait(full_bar(s), (it / S) & 1, abort_flag, p.timeout_ns);
        if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
        tc_fence_after();
        const uint32_t st = base + s * kDecStageBytes;
        if (ks < nks_main) {
          const uint32_t wsf = st + kDecWsfOff + lane * 16;
          const uint32_t xsf = st + kDecXsfOff + lane * 16;
          const uint32_t tsf = tmem + (static_cast<uint32_t>(q * 32) << 16) + kPairSfCol + s * kPairSlotCols;
          uint32_t r0[16], r1[16], rx[16];
#pragma unroll
          for (int kb = 0; kb < 4; ++kb) {       // tiles past the stage's last K block are never read
            const uint4 w0 = ld_shared_v4(wsf + kb * 512);
            const uint4 w1 = ld_shared_v4(wsf + 2048 + kb * 512);
            const uint4 x = ld_shared_v4(xsf + kb * 512);
            if constexpr (kSwiglu) {
              r0[4 * kb] = w0.x; r0[4 * kb + 1] = w0.y; r0[4 * kb + 2] = w1.x; r0[4 * kb + 3] = w1.y;
              r1[4 * kb] = w0.z; r1[4 * kb + 1] = w0.w; r1[4 * kb + 2] = w1.z; r1[4 * kb + 3] = w1.w;
            } else {
              r0[4 * kb] = w0.x; r0[4 * kb + 1] = w0.y; r0[4 * kb + 2] = w0.z; r0[4 * kb + 3] = w0.w;
              r1[4 * kb] = w1.x; r1[4 * kb + 1] = w1.y; r1[4 * kb + 2] = w1.z; r1[4 * kb + 3] = w1.w;
            }
            rx[4 * kb] = x.x; rx[4 * kb + 1] = x.y; rx[4 * kb + 2] = x.z; rx[4 * kb + 3] = x.w;
          }
          tmem_store16(tsf, r0);
          tmem_store16(tsf + 16, r1);
          tmem_store16(tsf + 32, rx);
          tmem_wait_st();
          tc_fence_before();
        } else if (my_row) {
          // R / G rounded to BF16 (as R * fp32(1 / G)), in place: this lane's
          // token row of each box (2 cw bytes)
          // (each lane starts at another 16-byte piece: the rows of a
          // quarter warp then fall in distinct banks)
          const int nj = min(cps, nch - (ks - nks_main) * cps);
          const int units = cw / 8, rot = (q * 32 + lane) >> (cw == 64 ? 0 : (cw == 32 ? 1 : 2));
          for (int j = 0; j < nj; ++j) {
            const uint32_t ad = st + j * rcb + (q * 32 + lane) * 2 * cw;
            for (int hh = 0; hh < units; ++hh) {
              const int h = (hh + rot) & (units - 1);
              const uint4 v = ld_shared_v4(ad + 16 * h);
              uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float lo = __fmul_rn(bf16_bits_to_float(w[i] & 0xFFFFu), Ginv);
                const float hi = __fmul_rn(bf16_bits_to_float(w[i] >> 16), Ginv);
                w[i] = pack_bf16x2(lo, hi);
              }
              st_shared_v4(ad + 16 * h, w[0], w[1], w[2], w[3]);
            }
          }
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(sf_full(s));
      }
    }
  } else if (warp >= 6) {
    // ----------------------------------------------------------- epilogue
    // Warp 6 + 4 hs + i reads TMEM lane quarter q = warp % 4 (weight rows
    // 32 q + lane of both halves) and accumulator columns [64 hs, 64 hs + 64)
    // (token rows), 32 at a time; both halves are read and rounded before
    // the accumulator is handed back.  Lane i stores its weight row's value
    // for each token row: a warp writes 64 contiguous bytes per row.
    const int q = warp & 3, hs = (warp - 6) >> 2;
    int tc = 0;
    for (int u = blockIdx.x; u < total; u += gridDim.x, ++tc) {
      int e, wrow, wb, row0, nrows;
      unit_of(u, e, wrow, wb, row0, nrows);
      if (!mbar_wait_cluster(acc_full, tc & 1, abort_flag, p.timeout_ns)) break;
      tc_fence_after();
      const float G = gscale_s[e];
      const int c0 = 64 * hs;                         // first token column of this warp
      const int nvalid = max(0, min(64, nrows - c0)); // token rows this warp stores
      uint32_t v0[2][16], v1[2][16];                  // BF16 pairs of consecutive token rows, per half
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        if (32 * c < nvalid) {
          uint32_t a[32], b[32];
          const uint32_t tacc = tmem + (static_cast<uint32_t>(q * 32) << 16) + c0 + 32 * c;
          tmem_load32(tacc, a);
          tmem_load32(tacc + 128, b);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            v0[c][j] = pack_bf16x2(__fmul_rn(__uint_as_float(a[2 * j]), G), __fmul_rn(__uint_as_float(a[2 * j + 1]), G));
            v1[c][j] = pack_bf16x2(__fmul_rn(__uint_as_float(b[2 * j]), G), __fmul_rn(__uint_as_float(b[2 * j + 1]), G));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
      const int feat = 32 * q + lane;
      if constexpr (!kSwiglu) {
        const int col = wb * kDecRowsPerUnit + feat;   // expert-local output column of half 0
        uint16_t* const y0 = p.y + static_cast<int64_t>(row0 + c0) * p.N + col;
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int t = 32 * c + j;
            if (t < nvalid) {
              const uint32_t w0 = v0[c][j >> 1], w1 = v1[c][j >> 1];
              y0[static_cast<int64_t>(t) * p.N] = static_cast<uint16_t>((j & 1) ? (w0 >> 16) : (w0 & 0xFFFFu));
              y0[static_cast<int64_t>(t) * p.N + 128] = static_cast<uint16_t>((j & 1) ? (w1 >> 16) : (w1 & 0xFFFFu));
            }
          }
      } else {
        const int Fh = p.N / 2;
        const int col = wb * (kDecRowsPerUnit / 2) + feat;   // h column
        uint16_t* const h0 = p.y + static_cast<int64_t>(row0 + c0) * Fh + col;
        unsigned int hmax = 0u;
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int t = 32 * c + 2 * j;
            if (t < nvalid) {
              const uint32_t o = swiglu_bf16x2(v0[c][j], v1[c][j]);
              h0[static_cast<int64_t>(t) * Fh] = static_cast<uint16_t>(o & 0xFFFFu);
              hmax = max(hmax, o & 0x7FFFu);
              if (t + 1 < nvalid) {
                h0[static_cast<int64_t>(t + 1) * Fh] = static_cast<uint16_t>(o >> 16);
                hmax = max(hmax, (o >> 16) & 0x7FFFu);
              }
            }
          }
        hmax = __reduce_max_sync(0xffffffffu, hmax);
        if (lane == 0 && hmax != 0u && p.amax_bits != nullptr) atomicMax(&p.amax_bits[e], hmax << 16);
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------------------
// W4A16 with the weights as the MMA's M operand, converted into TMEM.
//
// The trainer's GEMM Y = X . W_fq^T (X BF16; the weights given as NVFP4
// codes and scales, W_fq = bf16(fp32(val(q) val(s)) g_w[e])).  The 128 x N
// W4A16 kernel converts each weight tile into shared memory, where the MMA
// reads it back.  Here the converter warps store W_fq straight into tensor
// memory and the kind::f16 MMA reads it there as its A operand; only the
// BF16 row tile goes through shared memory to the tensor cores.  D^T = W .
// X^T: a unit is (expert, 128 weight rows, up to 256 of the expert's rows),
// the weight rows on the MMA's M (TMEM lanes) and the rows on its N = 256.
// A weight tile is converted once per 256 rows, and each MMA is the full
// 128 x 256 x 16.
//   stage       the codes of the unit's 128 weight rows for 64 K (128 x 32
//               bytes), their 512-byte scale tile, and the BF16 row tile
//               (256 rows x 64 K, 128-byte swizzle): 37 KB.
//   roles       warps 0 and 14 (lane 0) load the even and the odd stages
//               (two issuing threads fill a stage about twice as fast as
//               one); warp 1 lane 0 issues the MMAs; warps 2..5 convert the
//               even stages and warps 15..18 the odd ones (lane i of the
//               group's warp for quarter q: weight row 32 q + i), so that two
//               stages are converted at once; warps 6..13 the epilogue (warp
//               6 + 4 hs + q: lane quarter q, rows [128 hs, 128 hs + 128)).
//   TMEM        [0, 256) the accumulator (one buffer); [256, 512) eight A
//               slots of 32 columns (64 K of BF16, two per column).
//   pipeline    up to eight stages and eight A slots (slot it % 8): a stage
//               landing implies that its slot's previous MMAs have completed.
//   SwiGLU      a unit's 128 weight rows are one block of the interleaved
//               layout: 64 gate rows (lanes 0-63) and the matching 64 up
//               rows (lanes 64-127).  The up warps (quarters 2, 3) pass their
//               rounded values to the gate warps through shared memory
//               (bounded barrier waits), which apply SwiGLU: 64 h columns
//               per unit.
constexpr int kW16Rows = 128;                                  // weight rows per unit (M)
constexpr int kW16Tok = 256;                                   // expert rows per unit at most (N)
constexpr int kW16SfOff = kW16Rows * 32;                       // after the codes (64 K of FP4 per row)
constexpr int kW16XOff = kW16SfOff + 1024;                     // 5120: 1024-byte aligned row tile
constexpr int kW16StageBytes = kW16XOff + kW16Tok * 128;       // 37888
constexpr int kW16Slots = 8;                                   // A slots in TMEM
constexpr int kW16MaxStages = 8;
static_assert(kW16MaxStages <= kW16Slots, "a stage landing must imply its A slot is free");
constexpr int kW16ACol = 256;
constexpr int kW16ConvWarps = 4;                               // per group: even and odd stages
constexpr int kW16EpiWarp0 = 2 + kW16ConvWarps;                // 6
constexpr int kW16Loader1 = kW16EpiWarp0 + kDecEpiWarps;       // 14: the second loading warp
constexpr int kW16Conv1 = kW16Loader1 + 1;                     // 15: the odd stages' converters
constexpr int kW16Threads = 32 * (kW16Conv1 + kW16ConvWarps);  // 608
constexpr int kW16XchgBytes = 4 * 128 * 32 * 2;                // SwiGLU: four 8 KB up-to-gate buffers

template <bool kSwiglu>
__global__ void __launch_bounds__(kW16Threads, 1)
    grouped_gemm_w16m_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                             GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const base_ptr = smem_raw + (base - raw);
  const int S = p.stages;                         // <= kW16Slots
  const uint32_t xchg = base + S * kW16StageBytes;                          // kSwiglu only
  const uint32_t bar0 = xchg + (kSwiglu ? kW16XchgBytes : 0);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (S + s); };
  auto conv_full = [&](int j) { return bar0 + 8u * (2 * S + j); };               // A slot j converted
  auto x_full = [&](int k) { return bar0 + 8u * (2 * S + 2 * kW16Slots + k); };  // up values passed
  auto x_empty = [&](int k) { return bar0 + 8u * (2 * S + 2 * kW16Slots + 4 + k); };
  const uint32_t acc_full = bar0 + 8u * (2 * S + 2 * kW16Slots + 8);
  const uint32_t acc_empty = acc_full + 8;
  const uint32_t drain_bar = acc_full + 16;
  uint8_t* const misc = base_ptr + (drain_bar + 8 - base);
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(misc);
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  int32_t* const off_s = reinterpret_cast<int32_t*>(misc + 16);       // E + 1, clamped to rows_cap
  int32_t* const ub_s = off_s + p.E + 1;                                 // E + 1: first unit of each expert
  float* const gw_s = reinterpret_cast<float*>(ub_s + p.E + 1);         // g_w[e]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    prefetch_tensormap(&tm_x);
    prefetch_tensormap(&tm_w);
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int j = 0; j < kW16Slots; ++j) mbar_init(conv_full(j), kW16ConvWarps);   // one arrival per converter warp
    for (int k = 0; k < 4; ++k) {
      mbar_init(x_full(k), 1);
      mbar_init(x_empty(k), 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, kDecEpiWarps);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  const int nwb = p.N / kW16Rows;
  for (int i = threadIdx.x; i <= p.E; i += blockDim.x) {
    off_s[i] = min(p.expert_off[i], p.rows_cap);
    if (i < p.E) gw_s[i] = p.g_w[i];
  }
  __syncthreads();
  if (warp == 2) warp_block_prefix(ub_s, off_s, p.E, kW16Tok, nwb, lane);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int total = ub_s[p.E];
  const int nks = p.K / 64;                       // stages of 64 K
  const int n_col_tiles = p.K / 64;               // 128 x 4 scale tiles along K
  // units ordered expert, row block, weight block (weight blocks innermost:
  // the CTAs that run at the same time share a BF16 row tile, the larger
  // operand, and read it from L2; an expert's FP4 weights stay in L2 across
  // its row blocks)
  auto unit_of = [&](int u, int& e, int& wrow, int& wb, int& row0, int& nrows) {
    e = expert_of_row(ub_s, p.E, u);
    const int local = u - ub_s[e];
    const int tb = local / nwb;
    wb = local - tb * nwb;
    wrow = e * p.N + wb * kW16Rows;
    row0 = off_s[e] + kW16Tok * tb;
    nrows = min(kW16Tok, off_s[e + 1] - row0);
  };

  if ((warp == 0 || warp == kW16Loader1) && lane == 0) {
    // ---------------------------------------------------- producers (two)
    const int par = warp == 0 ? 0 : 1;            // the stages it % 2 == par
    int it = 0, last = -1;
    bool ok = true;
    for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
      int e, wrow, wb, row0, nrows;
      unit_of(u, e, wrow, wb, row0, nrows);
      for (int ks = 0; ks < nks; ++ks, ++it) {
        if ((it & 1) != par) continue;
        const int s = it % S;
        if (!mbar_wait(empty_bar(s), ((it / S) & 1) ^ 1u, abort_flag, p.timeout_ns)) { ok = false; break; }
        const uint32_t st = base + s * kW16StageBytes;
        mbar_expect_tx(full_bar(s), kW16SfOff + 512 + kW16Tok * 128);
        tma_load_2d(st, &tm_w, ks * 32, wrow, full_bar(s));                   // 128 rows x 32 bytes
        bulk_load(st + kW16SfOff, p.w_scales + (static_cast<int64_t>(wrow / 128) * n_col_tiles + ks) * 512, 512,
                  full_bar(s));
        tma_load_2d(st + kW16XOff, &tm_x, ks * 64, row0, full_bar(s));       // 256 rows x 64 BF16
        last = it;
      }
    }
    if (!ok)   // this thread's copies in flight land before the CTA exits
      for (int i = (last >= S ? last - S + 1 : 0); i <= last; ++i)
        if ((i & 1) == par) mbar_wait(full_bar(i % S), (i / S) & 1, nullptr, kDrainTimeoutNs);
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------------ MMA
    constexpr uint32_t kIdesc = idesc_bf16(kW16Tok);
    int it = 0, tc = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < total && ok; u += gridDim.x, ++tc) {
      if (!mbar_wait_cluster(acc_empty, (tc & 1) ^ 1u, abort_flag, p.timeout_ns)) { ok = false; break; }
      tc_fence_after();
      for (int ks = 0; ks < nks; ++ks, ++it) {
        const int s = it % S, j = it % kW16Slots;
        // the converters arrive after they saw the stage land: the row tile is there too
        if (!mbar_wait_cluster(conv_full(j), (it / kW16Slots) & 1, abort_flag, p.timeout_ns)) { ok = false; break; }
        tc_fence_after();
        const uint32_t st = base + s * kW16StageBytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)            // K = 16 per MMA, 32 bytes along the row tile's rows
          mma_bf16_tmem_a(tmem, tmem + kW16ACol + 32 * j + 8 * kk, desc_kmajor_sw128(st + kW16XOff + kk * 32), kIdesc,
                          (ks | kk) != 0 ? 1u : 0u);
        tc_commit(empty_bar(s));               // frees the stage (and, S <= 8 stages later, the A slot)
      }
      if (!ok) break;
      tc_commit(acc_full);
    }
    if (!ok) {
      tc_commit(drain_bar);
      mbar_wait(drain_bar, 0, nullptr, kDrainTimeoutNs);
    }
  } else if ((warp >= 2 && warp < kW16EpiWarp0) || warp >= kW16Conv1) {
    // ------------------------------------------------------------ converters
    // Lane i of the group's warp for quarter q: weight row 32 q + i of the
    // unit.  Its 32 code bytes and 4 scale bytes of the stage become 64 W_fq
    // values, stored as 32 columns of its TMEM lane in A slot it % 8 once the
    // stage has landed and the MMAs that last read the slot have completed.
    const int q = warp & 3;
    const int par = warp >= kW16Conv1 ? 1 : 0;   // the stages it % 2 == par
    const int r = 32 * q + lane;
    const uint32_t sf_off = kW16SfOff + (r & 31) * 16 + ((r >> 5) & 3) * 4;
    int it = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
      int e, wrow, wb, row0, nrows;
      unit_of(u, e, wrow, wb, row0, nrows);
      const float g = gw_s[e];
      for (int ks = 0; ks < nks; ++ks, ++it) {
        if ((it & 1) != par) continue;
        const int s = it % S, j = it % kW16Slots;
        // the stage landing implies that A slot j is free: the producer
        // refilled the stage after the MMAs of iteration it - S completed,
        // and those of it - 8 (the slot's last use) came before them
        const bool w_ok = mbar_wait(full_bar(s), (it / S) & 1, abort_flag, p.timeout_ns);
        if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
        tc_fence_after();
        const uint32_t st = base + s * kW16StageBytes;
        const uint4 c0 = ld_shared_v4(st + r * 32), c1 = ld_shared_v4(st + r * 32 + 16);
        const uint32_t sw = ld_shared_u32(st + sf_off);
        const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        const uint32_t ta = tmem + (static_cast<uint32_t>(q * 32) << 16) + kW16ACol + 32 * j;
#pragma unroll
        for (int hg = 0; hg < 2; ++hg) {          // 32 K (two blocks) per 16 columns
          uint32_t o[16];
#pragma unroll
          for (int b = 0; b < 2; ++b) {
            const int kb = 2 * hg + b;
            QCore qb{cw[2 * kb], cw[2 * kb + 1], (sw >> (8 * kb)) & 0xFFu, 0.0f};
            uint32_t w8[8];
            deq_block_bf16(qb, g, 1, w8);
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) o[8 * b + jj] = w8[jj];
          }
          tmem_store16(ta + 16 * hg, o);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(conv_full(j));
      }
    }
  } else if (warp >= kW16EpiWarp0 && warp < kW16Loader1) {
    // ----------------------------------------------------------- epilogue
    // Warp 6 + 4 hs + q reads lane quarter q (weight rows 32 q + lane) and
    // accumulator columns [128 hs, 128 hs + 128) (rows), rounded to BF16
    // before the accumulator is handed back.  Lane i stores its weight
    // row's value for each row: a warp writes 64 contiguous bytes per row.
    const int q = warp & 3, hs = (warp - kW16EpiWarp0) >> 2;
    const int pair = (q & 1) + 2 * hs;            // SwiGLU: gate warp q, up warp q + 2
    const uint32_t xb = xchg + pair * (128 * 32 * 2);
    int tc = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < total && ok; u += gridDim.x, ++tc) {
      int e, wrow, wb, row0, nrows;
      unit_of(u, e, wrow, wb, row0, nrows);
      if (!mbar_wait_cluster(acc_full, tc & 1, abort_flag, p.timeout_ns)) break;
      tc_fence_after();
      const int c0 = 128 * hs;
      const int nvalid = max(0, min(128, nrows - c0));   // rows this warp stores
      uint32_t v[4][16];                                  // BF16 pairs of consecutive rows
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if (32 * c < nvalid) {
          uint32_t a[32];
          tmem_load32(tmem + (static_cast<uint32_t>(q * 32) << 16) + c0 + 32 * c, a);
          tmem_wait_ld();
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) v[c][jj] = pack_bf16x2(__uint_as_float(a[2 * jj]), __uint_as_float(a[2 * jj + 1]));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
      if constexpr (!kSwiglu) {
        uint16_t* const y0 = p.y + static_cast<int64_t>(row0 + c0) * p.N + wb * kW16Rows + 32 * q + lane;
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) {
            const int t = 32 * c + jj;
            if (t < nvalid) {
              const uint32_t w = v[c][jj >> 1];
              y0[static_cast<int64_t>(t) * p.N] = static_cast<uint16_t>((jj & 1) ? (w >> 16) : (w & 0xFFFFu));
            }
          }
      } else if (q >= 2) {
        // up rows: hand the rounded values to the gate warp of the pair
        bool w_ok = mbar_wait(x_empty(pair), (tc & 1) ^ 1u, abort_flag, p.timeout_ns);
        if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) st_shared_u32(xb + ((16 * c + jj) * 32 + lane) * 4, v[c][jj]);
        __syncwarp();
        if (lane == 0) mbar_arrive(x_full(pair));
      } else {
        bool w_ok = mbar_wait(x_full(pair), tc & 1, abort_flag, p.timeout_ns);
        if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
        const int Fh = p.N / 2;
        // gate lane 32 q + i: h column wb * 64 + 32 q + i of the expert
        uint16_t* const h0 = p.y + static_cast<int64_t>(row0 + c0) * Fh + wb * (kW16Rows / 2) + 32 * q + lane;
        unsigned int hmax = 0u;
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            const int t = 32 * c + 2 * jj;
            const uint32_t up = ld_shared_u32(xb + ((16 * c + jj) * 32 + lane) * 4);
            if (t < nvalid) {
              const uint32_t o = swiglu_bf16x2(v[c][jj], up);
              h0[static_cast<int64_t>(t) * Fh] = static_cast<uint16_t>(o & 0xFFFFu);
              hmax = max(hmax, o & 0x7FFFu);
              if (t + 1 < nvalid) {
                h0[static_cast<int64_t>(t + 1) * Fh] = static_cast<uint16_t>(o >> 16);
                hmax = max(hmax, (o >> 16) & 0x7FFFu);
              }
            }
          }
        __syncwarp();
        if (lane == 0) mbar_arrive(x_empty(pair));
        hmax = __reduce_max_sync(0xffffffffu, hmax);
        if (lane == 0 && hmax != 0u && p.amax_bits != nullptr) atomicMax(&p.amax_bits[e], hmax << 16);
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// Per-expert amax for the FP4 compensation's residual:
// amax_r[e] = fp32(fp32(G_e / g_wc[e]) * 2688), G_e = fp32(g_a g_w[e]); the
// residual's decode scale times g_wc[e] is then G_e up to one rounding.
__global__ void fp4_comp_amax_kernel(const float* g_a, int g_a_per_expert, const float* g_w, const float* g_wc,
                                     int E, float* amax_r) {
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const float G = __fmul_rn(g_a[g_a_per_expert ? e : 0], g_w[e]);
    const float wc = g_wc[e];
    amax_r[e] = wc > 0.0f ? __fmul_rn(__fdiv_rn(G, wc), kNvfp4Range) : 0.0f;
  }
}

// One thread waits on a barrier that nothing completes; the bounded wait
// gives up after limit_ns and records the timeout.
__global__ void bounded_wait_selftest_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_addr(&bar), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    mbar_wait(smem_addr(&bar), 0, reinterpret_cast<volatile int*>(&abort_flag), limit_ns);
  }
}

// ------------------------------------------------------------------- host

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

int make_map_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t elem_bytes, uint64_t inner,
                uint64_t outer, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return set_error(QUADS_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * elem_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(QUADS_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return QUADS_OK;
}

// A 3D map over rows of `inner` elements grouped in blocks of 128 rows:
// dims (inner, 128 rows, blocks), box (box_inner, box_rows, box_blocks).
int make_map_3d_blocks(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t elem_bytes, uint64_t inner,
                       uint64_t rows, uint32_t box_inner, uint32_t box_rows, uint32_t box_blocks,
                       CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return set_error(QUADS_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  cuuint64_t dims[3] = {inner, 128, rows / 128};
  cuuint64_t strides[2] = {inner * elem_bytes, 128 * inner * elem_bytes};
  cuuint32_t box[3] = {box_inner, box_rows, box_blocks};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(QUADS_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return QUADS_OK;
}

// Channels per box of the wide and decode tiles' BF16 correction operands:
// the widest of 64, 32, 16 that divides n_chan (rows of 128, 64 or 32 bytes:
// fewer, longer rows per TMA copy).
int comp_box_channels(int n_chan) { return n_chan % 64 == 0 ? 64 : (n_chan % 32 == 0 ? 32 : 16); }
CUtensorMapSwizzle swizzle_of_row(int row_bytes) {
  return row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                          : (row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
}

// extra_words: the quantizing epilogue's tables (E + n_chan_h + N / 64 + 1)
size_t gemm_smem_bytes(int stages, int n_chan, int E, size_t extra_words = 0, int stage_b = kStageBytes,
                       int out_b = kOutStageBytes) {
  return 1024 + static_cast<size_t>(stages) * stage_b + static_cast<size_t>(n_chan / 16) * 2 * kCompChunkBytes +
         out_b + static_cast<size_t>(3 * stages + 9 + 2 * kSfSlots) * 8 + 16 +
         (static_cast<size_t>(2 * E + 1) + extra_words) * 4;
}

// FP4 compensation operands (device memory): the NVFP4 residual channels of
// the activations [rows_cap][Kc] and the weights' channel columns [E * N][Kc],
// codes row-major, scales tiled.
struct Fp4Comp {
  const uint8_t* a_codes;
  const uint8_t* a_scales;
  const uint8_t* w_codes;
  const uint8_t* w_scales;
  int64_t Kc;
};

// The quantizing epilogue's outputs (all device memory).
struct HQuant {
  const float* amax_in;
  const int32_t* chan;
  int n_chan;
  uint8_t* codes;
  uint8_t* scales;
  uint16_t* resid;
  float* g_out;
};

}  // namespace
}  // namespace quads

using namespace quads;

extern "C" {

}  // extern "C"

namespace quads {
namespace {

// Tile shape of the FP4 grouped GEMMs with the BF16 correction (or none)
// whose N is a multiple of 256 (quads_gemm_set_tile_shape): 0 = 128 x 128 on
// one CTA (the kernel above), 1 = 128 x 256 on one CTA, 2 = 256 x 256 on a
// pair of CTAs.  Other GEMMs always take the 128 x 128 kernel.
int g_tile_shape = 1;

size_t pair_smem_bytes(int stages, bool pair, int E, size_t extra_words) {
  return 1024 + static_cast<size_t>(stages) * wide_stage_bytes(pair) + pair_out_bytes() +
         static_cast<size_t>(2 * stages + 2 * kPairSfSlots + 3) * 8 + 16 +
         (static_cast<size_t>(4 * E + 2) + extra_words) * 4;
}

// Clusters of two that fit on the device at once with this much shared
// memory (one CTA per SM), cached per kernel instance.
template <bool kSwiglu, bool kQuant>
int pair_clusters(size_t smem) {
  static int cached = -1;
  static size_t cached_smem = 0;
  if (cached > 0 && cached_smem == smem) return cached;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(2 * (num_sms() / 2), 1, 1);
  cfg.blockDim = dim3(kPairThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr{};
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = 2;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, grouped_gemm_pair_kernel<kSwiglu, kQuant, true>, &cfg) != cudaSuccess ||
      n <= 0) {
    cudaGetLastError();
    n = num_sms() / 2;
  }
  cached = n;
  cached_smem = smem;
  return n;
}

template <bool kSwiglu, bool kQuant, bool kPair>
int launch_gemm_pair(const uint8_t* a_codes, const uint8_t* a_scales, const float* g_a, int g_a_per_expert,
                     const uint8_t* w_codes, const uint8_t* w_scales, const float* g_w, const int32_t* expert_off,
                     int E, int64_t rows_cap, int64_t N, int64_t K, const uint16_t* a_resid, const uint16_t* w_resid,
                     int n_chan, uint16_t* y, float* amax_out, cudaStream_t stream, const HQuant* hq) {
  CUtensorMap tm_a, tm_b, tm_r, tm_wc, tm_y;
  const uint32_t wrows = kPair ? 128 : 256;       // weight rows this CTA loads per tile
  QUADS_TRY(make_map_2d(&tm_a, a_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, rows_cap, kStageRowBytes, 128,
                        CU_TENSOR_MAP_SWIZZLE_128B));
  QUADS_TRY(make_map_2d(&tm_b, w_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, E * N, kStageRowBytes, wrows,
                        CU_TENSOR_MAP_SWIZZLE_128B));
  const int cw = comp_box_channels(n_chan);
  if (n_chan) {
    QUADS_TRY(make_map_2d(&tm_r, a_resid, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, n_chan, rows_cap, cw, 128,
                          swizzle_of_row(2 * cw)));
    QUADS_TRY(make_map_2d(&tm_wc, w_resid, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, n_chan, E * N, cw, wrows,
                          swizzle_of_row(2 * cw)));
  } else {
    tm_r = tm_a;
    tm_wc = tm_a;
  }
  if (y)
    QUADS_TRY(make_map_2d(&tm_y, y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kSwiglu ? N / 2 : N, rows_cap, 32, 32,
                          CU_TENSOR_MAP_SWIZZLE_64B));
  else
    tm_y = tm_a;                                  // never used: no h store
  const size_t extra = kQuant ? static_cast<size_t>(hq->n_chan + N / 64 + 1) : 0;
  const size_t smem_cap = 232448;
  int stages = kPair ? kMaxStages : kPairSfSlots;  // one CTA: a scale slot per stage
  while (stages >= 2 && pair_smem_bytes(stages, kPair, E, extra) > smem_cap) --stages;
  QUADS_REQUIRE(stages >= 2, QUADS_ERR_UNSUPPORTED_SHAPE, "not enough shared memory for two stages");
  const size_t smem = pair_smem_bytes(stages, kPair, E, extra);
  auto kernel = grouped_gemm_pair_kernel<kSwiglu, kQuant, kPair>;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
      cudaSuccess)
    return set_error(QUADS_ERR_CUDA, "cannot set %zu bytes of shared memory", smem);
  GemmParams p{};
  p.a_scales = a_scales;
  p.w_scales = w_scales;
  p.g_a = g_a;
  p.g_w = g_w;
  p.expert_off = expert_off;
  p.y = y;
  p.amax_bits = reinterpret_cast<unsigned int*>(amax_out);
  p.amax_h_in = kQuant ? hq->amax_in : nullptr;
  p.chan_h = kQuant ? hq->chan : nullptr;
  p.n_chan_h = kQuant ? hq->n_chan : 0;
  p.h_codes = kQuant ? hq->codes : nullptr;
  p.h_scales = kQuant ? hq->scales : nullptr;
  p.h_resid = kQuant ? hq->resid : nullptr;
  p.g_h_out = kQuant ? hq->g_out : nullptr;
  p.g_a_per_expert = g_a_per_expert ? 1 : 0;
  p.E = E;
  p.rows_cap = static_cast<int>(rows_cap);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.n_chan = n_chan;
  p.comp_cw = cw;
  p.stages = stages;
  p.timeout_ns = kGemmTimeoutNs;
  // at most one tile per 128 rows and 256 columns
  const int64_t max_tiles = (rows_cap / 128) * (N / PBN);
  if constexpr (kPair) {
    int64_t clusters = pair_clusters<kSwiglu, kQuant>(smem);
    if (sm_budget() > 0 && clusters > sm_budget() / 2) clusters = sm_budget() / 2 > 0 ? sm_budget() / 2 : 1;
    if (clusters > max_tiles) clusters = max_tiles;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(2 * clusters), 1, 1);
    cfg.blockDim = dim3(kPairThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr{};
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kernel, tm_a, tm_b, tm_r, tm_wc, tm_y, p) != cudaSuccess)
      return set_error(QUADS_ERR_CUDA, "launch of the pair-tile GEMM failed: %s",
                       cudaGetErrorString(cudaGetLastError()));
  } else {
    int64_t grid = grid_sms();
    if (grid > max_tiles) grid = max_tiles;
    kernel<<<static_cast<unsigned>(grid), kPairThreads, smem, stream>>>(tm_a, tm_b, tm_r, tm_wc, tm_y, p);
  }
  count_launches(1);
  return check_launch("grouped_gemm_pair_kernel");
}

// Average rows per expert at or below which the FP4 GEMMs with the BF16
// correction (or none), N % 256 == 0 and no fused quantization take the
// decode kernel (quads_gemm_set_decode_rows); 0: never.
int g_decode_rows = 64;

bool decode_selected(int64_t rows_cap, int E) {
  if (g_decode_rows <= 0) return false;
  const int64_t blocks = rows_cap / 128 - E;       // 128-row blocks beyond one padding block per expert
  const int64_t avg = (blocks > 0 ? blocks : 0) * 128 / E;
  return avg <= g_decode_rows;
}

size_t decode_smem_bytes(int stages, int E) {
  return 1024 + static_cast<size_t>(stages) * kDecStageBytes + static_cast<size_t>(3 * stages + 3) * 8 + 16 +
         static_cast<size_t>(3 * E + 2) * 4;
}

size_t w16m_smem_bytes(int stages, bool swiglu, int E) {
  return 1024 + static_cast<size_t>(stages) * kW16StageBytes + (swiglu ? kW16XchgBytes : 0) +
         static_cast<size_t>(2 * stages + 2 * kW16Slots + 8 + 3) * 8 + 16 + static_cast<size_t>(3 * E + 2) * 4;
}

// The W4A16 GEMM on the weights-as-M kernel (N % 256 == 0; arguments
// validated by launch_gemm).
template <bool kSwiglu>
int launch_gemm_w16m(const uint16_t* x, const uint8_t* w_codes, const uint8_t* w_scales, const float* g_w,
                     const int32_t* expert_off, int E, int64_t rows_cap, int64_t N, int64_t K, uint16_t* y,
                     float* amax_out, cudaStream_t stream) {
  CUtensorMap tm_x, tm_w;
  QUADS_TRY(make_map_2d(&tm_x, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, K, rows_cap, 64, kW16Tok,
                        CU_TENSOR_MAP_SWIZZLE_128B));
  QUADS_TRY(make_map_2d(&tm_w, w_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, E * N, 32, kW16Rows,
                        CU_TENSOR_MAP_SWIZZLE_NONE));
  const size_t smem_cap = 232448;
  int stages = kW16MaxStages;
  while (stages >= 2 && w16m_smem_bytes(stages, kSwiglu, E) > smem_cap) --stages;
  QUADS_REQUIRE(stages >= 2, QUADS_ERR_UNSUPPORTED_SHAPE, "not enough shared memory for two stages");
  const size_t smem = w16m_smem_bytes(stages, kSwiglu, E);
  auto kernel = grouped_gemm_w16m_kernel<kSwiglu>;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
      cudaSuccess)
    return set_error(QUADS_ERR_CUDA, "cannot set %zu bytes of shared memory", smem);
  GemmParams p{};
  p.w_scales = w_scales;
  p.g_w = g_w;
  p.expert_off = expert_off;
  p.y = y;
  p.amax_bits = reinterpret_cast<unsigned int*>(amax_out);
  p.E = E;
  p.rows_cap = static_cast<int>(rows_cap);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.stages = stages;
  p.timeout_ns = kGemmTimeoutNs;
  // at most one unit per 128 rows (segments are 128-aligned) and 128 weight rows
  const int64_t max_units = (rows_cap / 128) * (N / kW16Rows);
  int64_t grid = grid_sms();
  if (grid > max_units) grid = max_units;
  kernel<<<static_cast<unsigned>(grid), kW16Threads, smem, stream>>>(tm_x, tm_w, p);
  count_launches(1);
  return check_launch("grouped_gemm_w16m_kernel");
}

template <bool kSwiglu>
int launch_gemm_decode(const uint8_t* a_codes, const uint8_t* a_scales, const float* g_a, int g_a_per_expert,
                       const uint8_t* w_codes, const uint8_t* w_scales, const float* g_w, const int32_t* expert_off,
                       int E, int64_t rows_cap, int64_t N, int64_t K, const uint16_t* a_resid, const uint16_t* w_resid,
                       int n_chan, uint16_t* y, float* amax_out, cudaStream_t stream) {
  CUtensorMap tm_x, tm_w, tm_r, tm_wc;
  QUADS_TRY(make_map_2d(&tm_x, a_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, rows_cap, kStageRowBytes, kDecBox,
                        CU_TENSOR_MAP_SWIZZLE_128B));
  // weights: SwiGLU, the 64 gate (or up) rows of both 128-row blocks of a
  // unit in one 3D box; plain, the unit's 256 rows in one box
  if (kSwiglu)
    QUADS_TRY(make_map_3d_blocks(&tm_w, w_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, E * N, kStageRowBytes, 64, 2,
                                 CU_TENSOR_MAP_SWIZZLE_128B));
  else
    QUADS_TRY(make_map_2d(&tm_w, w_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, E * N, kStageRowBytes, 256,
                          CU_TENSOR_MAP_SWIZZLE_128B));
  const int cw = comp_box_channels(n_chan);
  if (n_chan) {
    QUADS_TRY(make_map_2d(&tm_r, a_resid, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, n_chan, rows_cap, cw, kDecBox,
                          swizzle_of_row(2 * cw)));
    if (kSwiglu)
      QUADS_TRY(make_map_3d_blocks(&tm_wc, w_resid, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, n_chan, E * N, cw, 64, 2,
                                   swizzle_of_row(2 * cw)));
    else
      QUADS_TRY(make_map_2d(&tm_wc, w_resid, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, n_chan, E * N, cw, 256,
                            swizzle_of_row(2 * cw)));
  } else {
    tm_r = tm_x;
    tm_wc = tm_x;
  }
  const size_t smem_cap = 232448;
  int stages = kDecSlots;
  while (stages >= 2 && decode_smem_bytes(stages, E) > smem_cap) --stages;
  QUADS_REQUIRE(stages >= 2, QUADS_ERR_UNSUPPORTED_SHAPE, "not enough shared memory for two stages");
  const size_t smem = decode_smem_bytes(stages, E);
  auto kernel = grouped_gemm_decode_kernel<kSwiglu>;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
      cudaSuccess)
    return set_error(QUADS_ERR_CUDA, "cannot set %zu bytes of shared memory", smem);
  GemmParams p{};
  p.a_scales = a_scales;
  p.w_scales = w_scales;
  p.g_a = g_a;
  p.g_w = g_w;
  p.expert_off = expert_off;
  p.y = y;
  p.amax_bits = reinterpret_cast<unsigned int*>(amax_out);
  p.g_a_per_expert = g_a_per_expert ? 1 : 0;
  p.E = E;
  p.rows_cap = static_cast<int>(rows_cap);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.n_chan = n_chan;
  p.comp_cw = cw;
  p.stages = stages;
  p.timeout_ns = kGemmTimeoutNs;
  // at most one unit per 128 rows (segments are 128-aligned) and 256 weight rows
  const int64_t max_units = (rows_cap / kDecTok) * (N / kDecRowsPerUnit);
  int64_t grid = grid_sms();
  if (grid > max_units) grid = max_units;
  kernel<<<static_cast<unsigned>(grid), kDecThreads, smem, stream>>>(tm_x, tm_w, tm_r, tm_wc, p);
  count_launches(1);
  return check_launch("grouped_gemm_decode_kernel");
}

template <bool kSwiglu, bool kQuant = false, bool kW4A16 = false, int kBN = BN>
int launch_gemm(const uint8_t* a_codes, const uint8_t* a_scales, const float* g_a, int g_a_per_expert,
                const uint8_t* w_codes, const uint8_t* w_scales, const float* g_w, const int32_t* expert_off, int E,
                int64_t rows_cap, int64_t N, int64_t K, const uint16_t* a_resid, const uint16_t* w_resid, int n_chan,
                uint16_t* y, float* amax_out, cudaStream_t stream, const HQuant* hq = nullptr,
                const Fp4Comp* fc = nullptr) {
  QUADS_REQUIRE(E >= 1 && E <= 256, QUADS_ERR_UNSUPPORTED_SHAPE, "E must be in [1, 256]");
  QUADS_REQUIRE(N > 0 && N % kBN == 0 && N <= (int64_t(1) << 20), QUADS_ERR_UNSUPPORTED_SHAPE,
                "N (%lld) must be a positive multiple of 128", (long long)N);
  QUADS_REQUIRE(K > 0 && K % 64 == 0 && K <= (int64_t(1) << 20), QUADS_ERR_UNSUPPORTED_SHAPE,
                "K (%lld) must be a positive multiple of 64", (long long)K);
  QUADS_REQUIRE(rows_cap >= 0 && rows_cap % BM == 0 && rows_cap < (int64_t(1) << 31), QUADS_ERR_INVALID_ARG,
                "rows_cap must be a multiple of 128");
  QUADS_REQUIRE(E * N < (int64_t(1) << 31), QUADS_ERR_UNSUPPORTED_SHAPE, "E * N too large");
  QUADS_REQUIRE(n_chan >= 0 && n_chan % 16 == 0 && n_chan <= kMaxChan, QUADS_ERR_UNSUPPORTED_SHAPE,
                "n_chan must be a multiple of 16 in [0, %d]", kMaxChan);
  QUADS_REQUIRE(a_codes && (kW4A16 || (a_scales && g_a)) && w_codes && w_scales && g_w && expert_off &&
                    (y || kQuant),
                QUADS_ERR_INVALID_ARG, "null pointer");
  if constexpr (kQuant) {
    QUADS_REQUIRE(hq && hq->amax_in && hq->codes && hq->scales && hq->g_out, QUADS_ERR_INVALID_ARG,
                  "amax_h_in, h_codes, h_scales and g_h_out are required");
    QUADS_REQUIRE(hq->n_chan >= 0 && hq->n_chan <= 256, QUADS_ERR_UNSUPPORTED_SHAPE, "n_chan_h must be in [0, 256]");
    QUADS_REQUIRE(hq->n_chan == 0 || (hq->chan && hq->resid), QUADS_ERR_INVALID_ARG, "chan_h and h_resid required");
    QUADS_REQUIRE(aligned(hq->codes, 16) && aligned(hq->scales, 16) && (!hq->resid || aligned(hq->resid, 4)),
                  QUADS_ERR_INVALID_ARG, "h_codes and h_scales must be 16-byte aligned");
  }
  QUADS_REQUIRE(n_chan == 0 || (a_resid && w_resid), QUADS_ERR_INVALID_ARG, "a_resid and w_resid required");
  if (fc) {
    QUADS_REQUIRE(n_chan == 0, QUADS_ERR_INVALID_ARG, "BF16 and FP4 compensation are exclusive");
    QUADS_REQUIRE(fc->Kc > 0 && fc->Kc % 64 == 0 && fc->Kc <= 1024, QUADS_ERR_UNSUPPORTED_SHAPE,
                  "Kc (%lld) must be a positive multiple of 64 up to 1024", (long long)fc->Kc);
    QUADS_REQUIRE(fc->a_codes && fc->a_scales && fc->w_codes && fc->w_scales && aligned(fc->a_codes, 16) &&
                      aligned(fc->w_codes, 16) && aligned(fc->a_scales, 16) && aligned(fc->w_scales, 16),
                  QUADS_ERR_INVALID_ARG, "FP4 compensation operands must be non-null and 16-byte aligned");
  }
  QUADS_REQUIRE(aligned(a_codes, 16) && aligned(w_codes, 16) && (kW4A16 || aligned(a_scales, 16)) &&
                    aligned(w_scales, 16) &&
                    (!y || aligned(y, 16)) && (n_chan == 0 || (aligned(a_resid, 16) && aligned(w_resid, 16))),
                QUADS_ERR_INVALID_ARG, "matrix pointers must be 16-byte aligned");
  if (kSwiglu && amax_out && cudaMemsetAsync(amax_out, 0, sizeof(float) * E, stream) != cudaSuccess)
    return set_error(QUADS_ERR_CUDA, "memset of amax_out failed");
  if (rows_cap == 0) return QUADS_OK;
  if constexpr (kW4A16 && kBN == 256 && !kQuant) {
    // the weights as M, converted into TMEM (tile shape 0 keeps the 128 x N kernel)
    if (g_tile_shape != 0 && N % 256 == 0)
      return launch_gemm_w16m<kSwiglu>(reinterpret_cast<const uint16_t*>(a_codes), w_codes, w_scales, g_w,
                                       expert_off, E, rows_cap, N, K, y, amax_out, stream);
  }
  if constexpr (!kW4A16 && kBN == BN && !kQuant) {
    if (fc == nullptr && N % kDecRowsPerUnit == 0 && decode_selected(rows_cap, E))
      return launch_gemm_decode<kSwiglu>(a_codes, a_scales, g_a, g_a_per_expert, w_codes, w_scales, g_w, expert_off,
                                         E, rows_cap, N, K, a_resid, w_resid, n_chan, y, amax_out, stream);
  }
  if constexpr (!kW4A16 && kBN == BN) {
    if (fc == nullptr && g_tile_shape != 0 && N % PBN == 0) {
      if (g_tile_shape == 2)
        return launch_gemm_pair<kSwiglu, kQuant, true>(a_codes, a_scales, g_a, g_a_per_expert, w_codes, w_scales,
                                                       g_w, expert_off, E, rows_cap, N, K, a_resid, w_resid, n_chan,
                                                       y, amax_out, stream, hq);
      return launch_gemm_pair<kSwiglu, kQuant, false>(a_codes, a_scales, g_a, g_a_per_expert, w_codes, w_scales, g_w,
                                                      expert_off, E, rows_cap, N, K, a_resid, w_resid, n_chan, y,
                                                      amax_out, stream, hq);
    }
  }

  CUtensorMap tm_a, tm_b, tm_r, tm_wc, tm_y;
  if (kW4A16) {
    // a_codes holds the BF16 activations [rows_cap][K]; W codes come in 32-byte rows per K = 64
    QUADS_TRY(make_map_2d(&tm_a, a_codes, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, K, rows_cap, 64, BM,
                          CU_TENSOR_MAP_SWIZZLE_128B));
    QUADS_TRY(make_map_2d(&tm_b, w_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, E * N, kMmaKBytes, kBN,
                          CU_TENSOR_MAP_SWIZZLE_NONE));
  } else {
    QUADS_TRY(make_map_2d(&tm_a, a_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, rows_cap, kStageRowBytes, BM,
                          CU_TENSOR_MAP_SWIZZLE_128B));
    QUADS_TRY(make_map_2d(&tm_b, w_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, E * N, kStageRowBytes, BN,
                          CU_TENSOR_MAP_SWIZZLE_128B));
  }
  if (n_chan) {
    QUADS_TRY(make_map_2d(&tm_r, a_resid, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, n_chan, rows_cap, 16, BM,
                          CU_TENSOR_MAP_SWIZZLE_32B));
    QUADS_TRY(make_map_2d(&tm_wc, w_resid, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, n_chan, E * N, 16, BN,
                          CU_TENSOR_MAP_SWIZZLE_32B));
  } else {
    tm_r = tm_a;
    tm_wc = tm_a;
  }
  if (y)
    QUADS_TRY(make_map_2d(&tm_y, y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kSwiglu ? N / 2 : N, rows_cap, 32, 32,
                          CU_TENSOR_MAP_SWIZZLE_64B));
  else
    tm_y = tm_a;                                  // never used: no h store
  CUtensorMap tm_a2 = tm_a, tm_b2 = tm_a;
  if (fc) {
    QUADS_TRY(make_map_2d(&tm_a2, fc->a_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, fc->Kc / 2, rows_cap, kMmaKBytes,
                          BM, CU_TENSOR_MAP_SWIZZLE_32B));
    QUADS_TRY(make_map_2d(&tm_b2, fc->w_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, fc->Kc / 2, E * N, kMmaKBytes, BN,
                          CU_TENSOR_MAP_SWIZZLE_32B));
  }
  const size_t extra = kQuant ? static_cast<size_t>(E + hq->n_chan + N / 64 + 1) : 0;
  const size_t smem_cap = 232448;   // 227 KB per block on sm_100
  int stages = kMaxStages;
  constexpr int kSB = stage_bytes(kW4A16, kBN);
  constexpr int kOB = out_stage_bytes(kQuant);
  while (stages >= 2 && gemm_smem_bytes(stages, n_chan, E, extra, kSB, kOB) > smem_cap) --stages;
  QUADS_REQUIRE(stages >= 2, QUADS_ERR_UNSUPPORTED_SHAPE, "not enough shared memory for two stages");
  const size_t smem = gemm_smem_bytes(stages, n_chan, E, extra, kSB, kOB);
  if (cudaFuncSetAttribute(grouped_gemm_kernel<kSwiglu, kQuant, kW4A16, kBN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return set_error(QUADS_ERR_CUDA, "cannot set %zu bytes of shared memory", smem);
  GemmParams p;
  p.a_scales = a_scales;
  p.w_scales = w_scales;
  p.g_a = g_a;
  p.g_w = g_w;
  p.expert_off = expert_off;
  p.y = y;
  p.amax_bits = reinterpret_cast<unsigned int*>(amax_out);
  p.amax_h_in = kQuant ? hq->amax_in : nullptr;
  p.chan_h = kQuant ? hq->chan : nullptr;
  p.n_chan_h = kQuant ? hq->n_chan : 0;
  p.h_codes = kQuant ? hq->codes : nullptr;
  p.h_scales = kQuant ? hq->scales : nullptr;
  p.h_resid = kQuant ? hq->resid : nullptr;
  p.g_h_out = kQuant ? hq->g_out : nullptr;
  p.a2_scales = fc ? fc->a_scales : nullptr;
  p.w2_scales = fc ? fc->w_scales : nullptr;
  p.nkb_comp = fc ? static_cast<int>(fc->Kc / 64) : 0;
  p.g_a_per_expert = g_a_per_expert ? 1 : 0;
  p.E = E;
  p.rows_cap = static_cast<int>(rows_cap);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.n_chan = n_chan;
  p.comp_cw = 16;                                 // this kernel's correction boxes are 16 channels wide
  p.stages = stages;
  p.timeout_ns = kGemmTimeoutNs;
  const int64_t max_tiles = (rows_cap / BM) * (N / kBN);
  int grid = grid_sms();
  if (grid > max_tiles) grid = static_cast<int>(max_tiles);
  grouped_gemm_kernel<kSwiglu, kQuant, kW4A16, kBN><<<grid, threads_for(kQuant, kW4A16), smem, stream>>>(
      tm_a, tm_b, tm_r, tm_wc, tm_y, tm_a2, tm_b2, p);
  count_launches(1);
  return check_launch("grouped_gemm_kernel");
}

}  // namespace
}  // namespace quads

extern "C" {

int quads_moe_grouped_gemm_nvfp4(const uint8_t* a_codes, const uint8_t* a_scales, const float* g_a,
                                 int g_a_per_expert, const uint8_t* w_codes, const uint8_t* w_scales, const float* g_w,
                                 const int32_t* expert_off, int E, int64_t rows_cap, int64_t N, int64_t K,
                                 const uint16_t* a_resid, const uint16_t* w_resid, int n_chan, uint16_t* y,
                                 quads_stream_t stream) {
  clear_error();
  return launch_gemm<false>(a_codes, a_scales, g_a, g_a_per_expert, w_codes, w_scales, g_w, expert_off, E, rows_cap,
                            N, K, a_resid, w_resid, n_chan, y, nullptr, stream);
}

int quads_moe_grouped_gemm_nvfp4_fp4comp(const uint8_t* a_codes, const uint8_t* a_scales, const float* g_a,
                                         int g_a_per_expert, const uint8_t* w_codes, const uint8_t* w_scales,
                                         const float* g_w, const int32_t* expert_off, int E, int64_t rows_cap,
                                         int64_t N, int64_t K, const uint8_t* r_codes, const uint8_t* r_scales,
                                         const uint8_t* wc_codes, const uint8_t* wc_scales, int64_t Kc, uint16_t* y,
                                         quads_stream_t stream) {
  clear_error();
  const Fp4Comp fc{r_codes, r_scales, wc_codes, wc_scales, Kc};
  return launch_gemm<false>(a_codes, a_scales, g_a, g_a_per_expert, w_codes, w_scales, g_w, expert_off, E, rows_cap,
                            N, K, nullptr, nullptr, 0, y, nullptr, stream, nullptr, &fc);
}

int quads_moe_grouped_gemm_nvfp4_swiglu_fp4comp(const uint8_t* a_codes, const uint8_t* a_scales, const float* g_a,
                                                int g_a_per_expert, const uint8_t* w_codes, const uint8_t* w_scales,
                                                const float* g_w, const int32_t* expert_off, int E, int64_t rows_cap,
                                                int64_t F, int64_t K, const uint8_t* r_codes,
                                                const uint8_t* r_scales, const uint8_t* wc_codes,
                                                const uint8_t* wc_scales, int64_t Kc, uint16_t* h, float* amax_out,
                                                quads_stream_t stream) {
  clear_error();
  QUADS_REQUIRE(F > 0 && F % 64 == 0, QUADS_ERR_UNSUPPORTED_SHAPE, "F (%lld) must be a positive multiple of 64",
                (long long)F);
  const Fp4Comp fc{r_codes, r_scales, wc_codes, wc_scales, Kc};
  return launch_gemm<true>(a_codes, a_scales, g_a, g_a_per_expert, w_codes, w_scales, g_w, expert_off, E, rows_cap,
                           2 * F, K, nullptr, nullptr, 0, h, amax_out, stream, nullptr, &fc);
}

int quads_moe_grouped_gemm_w4a16(const uint16_t* x, const uint8_t* w_codes, const uint8_t* w_scales,
                                 const float* g_w, const int32_t* expert_off, int E, int64_t rows_cap, int64_t N,
                                 int64_t K, uint16_t* y, quads_stream_t stream) {
  clear_error();
  // 256 weight rows per tile where N allows: half the activation traffic per FLOP
  const uint8_t* xa = reinterpret_cast<const uint8_t*>(x);
  if (N % 256 == 0)
    return launch_gemm<false, false, true, 256>(xa, nullptr, nullptr, 0, w_codes, w_scales, g_w, expert_off, E,
                                                rows_cap, N, K, nullptr, nullptr, 0, y, nullptr, stream);
  return launch_gemm<false, false, true>(xa, nullptr, nullptr, 0, w_codes, w_scales, g_w, expert_off, E, rows_cap, N,
                                         K, nullptr, nullptr, 0, y, nullptr, stream);
}

int quads_moe_grouped_gemm_w4a16_swiglu(const uint16_t* x, const uint8_t* w_codes, const uint8_t* w_scales,
                                        const float* g_w, const int32_t* expert_off, int E, int64_t rows_cap,
                                        int64_t F, int64_t K, uint16_t* h, float* amax_out, quads_stream_t stream) {
  clear_error();
  QUADS_REQUIRE(F > 0 && F % 64 == 0, QUADS_ERR_UNSUPPORTED_SHAPE, "F (%lld) must be a positive multiple of 64",
                (long long)F);
  const uint8_t* xa = reinterpret_cast<const uint8_t*>(x);
  if (F % 128 == 0)
    return launch_gemm<true, false, true, 256>(xa, nullptr, nullptr, 0, w_codes, w_scales, g_w, expert_off, E,
                                               rows_cap, 2 * F, K, nullptr, nullptr, 0, h, amax_out, stream);
  return launch_gemm<true, false, true>(xa, nullptr, nullptr, 0, w_codes, w_scales, g_w, expert_off, E, rows_cap,
                                        2 * F, K, nullptr, nullptr, 0, h, amax_out, stream);
}

int quads_moe_fp4_comp_amax(const float* g_a, int g_a_per_expert, const float* g_w, const float* g_wc, int E,
                            float* amax_r, quads_stream_t stream) {
  clear_error();
  QUADS_REQUIRE(E >= 1 && E <= 4096, QUADS_ERR_UNSUPPORTED_SHAPE, "E must be in [1, 4096]");
  QUADS_REQUIRE(g_a && g_w && g_wc && amax_r, QUADS_ERR_INVALID_ARG, "null pointer");
  fp4_comp_amax_kernel<<<1, 256, 0, stream>>>(g_a, g_a_per_expert, g_w, g_wc, E, amax_r);
  count_launches(1);
  return check_launch("fp4_comp_amax_kernel");
}

int quads_moe_grouped_gemm_nvfp4_swiglu_quant(const uint8_t* a_codes, const uint8_t* a_scales, const float* g_a,
                                              int g_a_per_expert, const uint8_t* w_codes, const uint8_t* w_scales,
                                              const float* g_w, const int32_t* expert_off, int E, int64_t rows_cap,
                                              int64_t F, int64_t K, const uint16_t* a_resid,
                                              const uint16_t* w_resid, int n_chan, const float* amax_h_in,
                                              const int32_t* chan_h, int n_chan_h, uint8_t* h_codes,
                                              uint8_t* h_scales, uint16_t* h_resid, float* g_h_out,
                                              float* amax_h_out, uint16_t* h, quads_stream_t stream) {
  clear_error();
  QUADS_REQUIRE(F > 0 && F % 64 == 0, QUADS_ERR_UNSUPPORTED_SHAPE, "F (%lld) must be a positive multiple of 64",
                (long long)F);
  const HQuant hq{amax_h_in, chan_h, n_chan_h, h_codes, h_scales, h_resid, g_h_out};
  return launch_gemm<true, true>(a_codes, a_scales, g_a, g_a_per_expert, w_codes, w_scales, g_w, expert_off, E,
                                 rows_cap, 2 * F, K, a_resid, w_resid, n_chan, h, amax_h_out, stream, &hq);
}

int quads_moe_grouped_gemm_nvfp4_swiglu(const uint8_t* a_codes, const uint8_t* a_scales, const float* g_a,
                                        int g_a_per_expert, const uint8_t* w_codes, const uint8_t* w_scales,
                                        const float* g_w, const int32_t* expert_off, int E, int64_t rows_cap,
                                        int64_t F, int64_t K, const uint16_t* a_resid, const uint16_t* w_resid,
                                        int n_chan, uint16_t* h, float* amax_out, quads_stream_t stream) {
  clear_error();
  QUADS_REQUIRE(F > 0 && F % 64 == 0, QUADS_ERR_UNSUPPORTED_SHAPE, "F (%lld) must be a positive multiple of 64",
                (long long)F);
  return launch_gemm<true>(a_codes, a_scales, g_a, g_a_per_expert, w_codes, w_scales, g_w, expert_off, E, rows_cap,
                           2 * F, K, a_resid, w_resid, n_chan, h, amax_out, stream);
}

int quads_gemm_set_tile_shape(int shape) {
  clear_error();
  QUADS_REQUIRE(shape >= 0 && shape <= 2, QUADS_ERR_INVALID_ARG, "tile shape must be 0, 1 or 2");
  const int prev = g_tile_shape;
  g_tile_shape = shape;
  return prev;
}

int quads_gemm_set_decode_rows(int rows) {
  clear_error();
  QUADS_REQUIRE(rows >= 0, QUADS_ERR_INVALID_ARG, "decode rows must be >= 0");
  const int prev = g_decode_rows;
  g_decode_rows = rows;
  return prev;
}

int quads_device_status(quads_stream_t stream) {
  clear_error();
  if (cudaStreamSynchronize(stream) != cudaSuccess)
    return set_error(QUADS_ERR_CUDA, "stream synchronize failed: %s", cudaGetErrorString(cudaGetLastError()));
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_wait_status, sizeof(v)) != cudaSuccess)
    return set_error(QUADS_ERR_CUDA, "cannot read the device status word");
  if (v) {
    unsigned int zero = 0;
    if (cudaMemcpyToSymbol(g_wait_status, &zero, sizeof(zero)) != cudaSuccess)
      return set_error(QUADS_ERR_CUDA, "cannot clear the device status word");
    return set_error(QUADS_ERR_TIMEOUT, "a device-side wait timed out");
  }
  return QUADS_OK;
}

int quads_selftest_bounded_wait(uint64_t timeout_ns, quads_stream_t stream) {
  clear_error();
  QUADS_REQUIRE(timeout_ns > 0 && timeout_ns <= 10000000000ull, QUADS_ERR_INVALID_ARG,
                "timeout must be in (0, 10 s]");
  bounded_wait_selftest_kernel<<<1, 32, 0, stream>>>(timeout_ns);
  count_launches(1);
  return check_launch("bounded_wait_selftest_kernel");
}

}  // extern "C"
