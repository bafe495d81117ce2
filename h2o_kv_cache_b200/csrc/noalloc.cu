// Allocation-free attention with summed attention weights (h2o_attend_noalloc).
//
// Some callers cannot call cudaMalloc: a serving engine that reserves nearly
// all of the GPU's memory for its own pool up front has none left to give, and
// latency-critical code cannot afford cudaMalloc's implicit device
// synchronisation.  This entry point therefore takes every input and output
// from the caller and keeps its only scratch -- the fixed-point accumulator
// rows of the summed weights and the device error word -- in a fixed-size
// array defined here at file scope.  Each GPU that loads the library holds that array until the process
// exits.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <mutex>

#include "../../include/h2o.h"
#include "h2o_internal.cuh"

namespace {

// 16 MiB: 2 Mi 64-bit accumulator words (one row of M + S per (b, KV head)),
// then the error word.
constexpr size_t kScratchWords = (size_t)2 << 20;
constexpr size_t kScratchBytes = kScratchWords * sizeof(unsigned long long) + 256;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

// Device address of g_scratch per device.  In host code the name g_scratch is
// only a host-side stand-in, so the address is looked up once per device with
// that device current, then passed to the kernels.
constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

int set_err(int code, const char* msg) {
  char buf[512];
  snprintf(buf, sizeof(buf), "h2o_attend_noalloc: %s", msg);
  return h2o::set_thread_error(code, buf);   // read back with h2o_last_error(NULL)
}

cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

// colsum[bh, c] for c < M: the slot's summed weight (0 for slots >= n_valid);
// colsum[bh, M + j]: chunk key j's summed weight; from the accumulator rows.
__global__ void colsum_kernel(const unsigned long long* __restrict__ acc, float* __restrict__ colsum,
                              int64_t S, int64_t M, int64_t stride, float fx_inv) {
  const int bh = blockIdx.y;
  const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t ncol = M + S;
  if (c >= ncol) return;
  colsum[(int64_t)bh * ncol + c] = h2o::colsum_value(acc[(int64_t)bh * stride + c], fx_inv);
}

}  // namespace

extern "C" int h2o_attend_noalloc(const void* q, const void* k, const void* v, const void* k_cache,
                                  const void* v_cache, int B, int Hq, int Hkv, int d, int dtype,
                                  int64_t M, int64_t n_valid, int64_t S, void* out, float* colsum,
                                  void* stream) {
  if (!q || !k || !v || !out || !colsum) return set_err(H2O_EINVAL, "NULL input or output");
  if (n_valid > 0 && (!k_cache || !v_cache)) return set_err(H2O_EINVAL, "NULL cache with n_valid > 0");
  if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || (d != 64 && d != 128) ||
      (dtype != H2O_F32 && dtype != H2O_BF16) || S < 1 || M < 0 || n_valid < 0 || n_valid > M)
    return set_err(H2O_EINVAL, "bad sizes");
  const bool umma = h2o::attn_umma_supported(dtype, d);
  const int G = Hq / Hkv;
  const int64_t stride = (M + S + 3) & ~(int64_t)3;   // accumulator words per (b, KV head)
  const double need = (double)B * Hkv * (double)stride;
  if (need > (double)kScratchWords) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "problem needs %.0f scratch words, above the fixed maximum of %zu "
             "(B*Hkv*(M+S rounded up to a multiple of 4) must be <= %zu)",
             need, kScratchWords, kScratchWords);
    return set_err(H2O_ESHAPE, msg);
  }
  void* base = nullptr;
  cudaError_t e = scratch_address(&base);
  if (e != cudaSuccess) return set_err(H2O_ECUDA, cudaGetErrorString(e));
  unsigned long long* acc = static_cast<unsigned long long*>(base);
  int* err = reinterpret_cast<int*>(static_cast<unsigned char*>(base) +
                                    kScratchWords * sizeof(unsigned long long));
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  // The accumulator rows and the error word must start at zero: the array
  // keeps whatever the previous call left.
  e = cudaMemsetAsync(acc, 0, (size_t)need * sizeof(unsigned long long), st);
  if (e == cudaSuccess) e = cudaMemsetAsync(err, 0, sizeof(int), st);
  if (e != cudaSuccess) return set_err(H2O_ECUDA, cudaGetErrorString(e));

  h2o::AttnArgs a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.out = out;
  a.kc = k_cache;
  a.vc = v_cache;
  a.colacc = acc;
  a.err = err;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.d = d;
  a.S = S;
  a.M = M;
  a.n_valid = n_valid;
  a.acc_stride = stride;
  a.scale = (float)(1.0 / std::sqrt((double)d));
  a.fx_shift = h2o::colsum_shift(S, G);
  e = umma ? h2o::launch_attn_umma(a, false, st) : h2o::launch_attn_simt(a, dtype, false, st);
  if (e != cudaSuccess) return set_err(H2O_ECUDA, cudaGetErrorString(e));
  const int threads = 256;
  dim3 grid((unsigned)((M + S + threads - 1) / threads), (unsigned)(B * Hkv));
  colsum_kernel<<<grid, threads, 0, st>>>(acc, colsum, S, M, stride, h2o::fx_inv_of(a.fx_shift));
  e = cudaGetLastError();
  if (e != cudaSuccess) return set_err(H2O_ECUDA, cudaGetErrorString(e));
  return H2O_OK;
}
