// Allocation-free attention with summed attention weights (h2o_attend_noalloc).
//
// Some callers cannot call cudaMalloc: a serving engine that reserves nearly
// all of the GPU's memory for its own pool up front has none left to give, and
// latency-critical code cannot afford cudaMalloc's implicit device
// synchronisation.  This entry point therefore takes every input and output
// from the caller and keeps its only scratch -- the per-row-tile partial column
// sums and the device error word -- in a fixed-size array defined here at file
// scope.  Each GPU that loads the library holds that array until the process
// exits.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <mutex>

#include "../../include/h2o.h"
#include "h2o_internal.cuh"

namespace {

// 16 MiB: 4 Mi floats of partial column sums, then the error word.
constexpr size_t kScratchFloats = (size_t)4 << 20;
constexpr size_t kScratchBytes = kScratchFloats * sizeof(float) + 256;

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
// colsum[bh, M + j]: chunk key j's summed weight.  Fixed-order sums of the
// attention kernel's partial rows.
__global__ void colsum_kernel(const float* __restrict__ partials, float* __restrict__ colsum, int G,
                              int64_t S, int64_t M, int64_t n_valid, int row_tile, int64_t stride) {
  const int bh = blockIdx.y;
  const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t ncol = M + S;
  if (c >= ncol) return;
  const int n_rt = (int)((S + row_tile - 1) / row_tile);
  const float* base = partials + (int64_t)bh * (G * n_rt) * stride;
  float acc = 0.f;
  if (c < M) {
    if (c < n_valid)
      for (int t = 0; t < G * n_rt; ++t) acc += base[(int64_t)t * stride + c];
  } else {
    const int64_t j = c - M;
    const int rt0 = (int)(j / row_tile);
    for (int gl = 0; gl < G; ++gl)
      for (int rt = rt0; rt < n_rt; ++rt) acc += base[(int64_t)(gl * n_rt + rt) * stride + c];
  }
  colsum[(int64_t)bh * ncol + c] = acc;
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
  const int row_tile = umma ? h2o::kUmmaRowTile : h2o::kSimtRowTile;
  const int G = Hq / Hkv;
  const int64_t n_rt = (S + row_tile - 1) / row_tile;
  const int64_t stride = h2o::partial_stride(M, S);
  const double need = (double)B * Hkv * G * n_rt * (double)stride;
  if (need > (double)kScratchFloats) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "problem needs %.0f scratch floats, above the fixed maximum of %zu "
             "(B*Hkv*(Hq/Hkv)*ceil(S/%d)*(M+S rounded up to a multiple of 4) must be <= %zu)",
             need, kScratchFloats, row_tile, kScratchFloats);
    return set_err(H2O_ESHAPE, msg);
  }
  void* base = nullptr;
  cudaError_t e = scratch_address(&base);
  if (e != cudaSuccess) return set_err(H2O_ECUDA, cudaGetErrorString(e));
  float* partials = static_cast<float*>(base);
  int* err = reinterpret_cast<int*>(static_cast<unsigned char*>(base) + kScratchFloats * sizeof(float));
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  // The error word must start at zero; the partials need no clearing (the
  // column sums read only entries the attention kernel wrote in this call).
  e = cudaMemsetAsync(err, 0, sizeof(int), st);
  if (e != cudaSuccess) return set_err(H2O_ECUDA, cudaGetErrorString(e));

  h2o::AttnArgs a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.out = out;
  a.kc = k_cache;
  a.vc = v_cache;
  a.partials = partials;
  a.err = err;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.d = d;
  a.S = S;
  a.M = M;
  a.n_valid = n_valid;
  a.part_stride = stride;
  a.scale = (float)(1.0 / std::sqrt((double)d));
  e = umma ? h2o::launch_attn_umma(a, false, st) : h2o::launch_attn_simt(a, dtype, false, st);
  if (e != cudaSuccess) return set_err(H2O_ECUDA, cudaGetErrorString(e));
  const int threads = 256;
  dim3 grid((unsigned)((M + S + threads - 1) / threads), (unsigned)(B * Hkv));
  colsum_kernel<<<grid, threads, 0, st>>>(partials, colsum, h2o::partial_groups(G, umma), S, M,
                                           n_valid, row_tile, stride);
  e = cudaGetLastError();
  if (e != cudaSuccess) return set_err(H2O_ECUDA, cudaGetErrorString(e));
  return H2O_OK;
}
