// Host-side error state of the svg_b200 library.
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdio.h>

#include <atomic>
#include <mutex>

#include "common.cuh"

namespace svg {

static thread_local char g_last_error[512] = "";

svg_status fail(svg_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return st;
}

void clear_error() { g_last_error[0] = '\0'; }

svg_status check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SVG_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return SVG_OK;
}

int sm_count() {
  static std::mutex mu;
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  std::lock_guard<std::mutex> lk(mu);
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

static std::atomic<uint32_t> g_wait_limit{kDefaultWaitLimit};

uint32_t wait_limit() { return g_wait_limit.load(std::memory_order_relaxed); }

}  // namespace svg

extern "C" const char* svg_last_error(void) { return svg::g_last_error; }

extern "C" svg_status svg_set_wait_limit(uint32_t polls) {
  svg::clear_error();
  svg::g_wait_limit.store(polls == 0 ? svg::kDefaultWaitLimit : polls, std::memory_order_relaxed);
  return SVG_OK;
}

extern "C" uint32_t svg_get_wait_limit(void) { return svg::wait_limit(); }

extern "C" const char* svg_version(void) { return "svg_b200 0.1 sm_100a"; }
