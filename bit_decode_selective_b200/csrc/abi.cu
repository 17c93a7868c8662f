// abi.cu -- status strings, error messages and buffer-size queries of the C ABI.
#include <cstring>
#include <mutex>

#include "common.cuh"

namespace sf {

static thread_local char g_err[512] = "";

void set_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
}

void clear_error() { g_err[0] = 0; }

int num_sms() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

}  // namespace sf

extern "C" {

int sf_abi_version(void) { return SF_ABI_VERSION; }

const char* sf_status_string(sf_status st) {
  switch (st) {
    case SF_OK: return "ok";
    case SF_ERR_INVALID_ARG: return "invalid argument";
    case SF_ERR_UNSUPPORTED: return "unsupported configuration";
    case SF_ERR_CUDA: return "CUDA error";
    case SF_ERR_TIMEOUT: return "timed out";
    case SF_ERR_WORKSPACE: return "workspace too small";
  }
  return "unknown status";
}

const char* sf_last_error(void) { return sf::g_err; }

sf_status sf_wq_bytes(int n, int k, int b, int r, int group, size_t* base_bytes,
                      size_t* refine_bytes, size_t* sz_bytes) {
  SF_REQUIRE(n > 0 && k > 0 && group > 0 && k % group == 0, "bad shape n=%d k=%d group=%d", n, k,
             group);
  SF_REQUIRE(b >= 2 && b <= 4 && r >= 1 && r <= 2, "bad bits b=%d r=%d", b, r);
  if (base_bytes) *base_bytes = (size_t)n * k * b / 8;
  if (refine_bytes) *refine_bytes = (size_t)k * n * r / 8;
  if (sz_bytes) *sz_bytes = (size_t)n * (k / group) * 2 * sizeof(uint16_t);
  return SF_OK;
}

sf_status sf_kv_bytes(int batch, int h_kv, int d, int t_max, int b, int r, int group,
                      size_t* code_bytes, size_t* refine_bytes, size_t* sz_bytes) {
  SF_REQUIRE(batch > 0 && h_kv > 0 && d > 0 && t_max > 0 && group > 0 && d % group == 0,
             "bad KV shape");
  SF_REQUIRE(b >= 2 && b <= 4 && (r == 1 || r == 2), "bad KV bits b=%d r=%d", b, r);
  size_t tok = (size_t)batch * h_kv * t_max;
  if (code_bytes) *code_bytes = tok * d * b / 8;
  if (refine_bytes) *refine_bytes = tok * d * r / 8;
  if (sz_bytes) *sz_bytes = tok * (d / group) * 2 * sizeof(uint16_t);
  return SF_OK;
}

}  // extern "C"
