// Error reporting, launch accounting and device queries shared by all entry points.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <mutex>

#include "common.cuh"

namespace quads {

namespace {
thread_local char g_last_error[512] = "";
std::atomic<uint64_t> g_launches{0};
std::mutex g_sm_mutex;
int g_sm_count[64] = {0};
std::atomic<int> g_sm_budget{0};
}  // namespace

int set_error(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return code;
}

void clear_error() { g_last_error[0] = '\0'; }

void count_launches(uint64_t n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

int check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(QUADS_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return QUADS_OK;
}

int num_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  std::lock_guard<std::mutex> lock(g_sm_mutex);
  if (g_sm_count[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    g_sm_count[dev] = n;
  }
  return g_sm_count[dev];
}

int sm_budget() {
  const int b = g_sm_budget.load(std::memory_order_relaxed);
  const int n = num_sms();
  return b > 0 && b < n ? b : 0;
}

int grid_sms() {
  const int b = sm_budget();
  return b > 0 ? b : num_sms();
}

int persistent_grid(const void* kernel, int threads, size_t smem, int64_t work_blocks) {
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem) != cudaSuccess || per_sm < 1)
    per_sm = 1;
  int64_t cap = static_cast<int64_t>(per_sm) * num_sms();
  int64_t g = work_blocks < cap ? work_blocks : cap;
  return static_cast<int>(g < 1 ? 1 : g);
}

}  // namespace quads

extern "C" {

const char* quads_last_error(void) { return quads::g_last_error; }

int quads_abi_version(void) { return 1; }

uint64_t quads_launch_count(void) { return quads::g_launches.load(); }

int quads_set_sm_budget(int n) {
  quads::clear_error();
  QUADS_REQUIRE(n >= 0, QUADS_ERR_INVALID_ARG, "the SM budget must be >= 0");
  return quads::g_sm_budget.exchange(n);
}

size_t quads_scales_bytes(int64_t rows, int64_t K, int scale_layout) {
  if (rows < 0 || K < 0 || K % 16 != 0) return 0;
  if (scale_layout != QUADS_SCALES_LINEAR && scale_layout != QUADS_SCALES_TILED) return 0;
  return static_cast<size_t>(quads::scale_bytes(rows, K, scale_layout));
}

}  // extern "C"
