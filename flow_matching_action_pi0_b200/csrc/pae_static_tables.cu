// pae_precompute_tables_static: the timestep/modulation table build without a
// context and without any device allocation.
//
// Who needs it: callers that may not allocate device memory once they are
// running.  A real-time control process that has finished its set-up and must
// not call cudaMalloc (it can synchronise the device and stall the control
// loop), a host framework that owns all device memory through its own arena,
// or code that is capturing a stream into a CUDA graph, where cudaMalloc is not
// allowed.  Such callers cannot create a pae context (pae_create allocates its
// buffers), but they can still turn a timestep grid into the same fp32
// modulation tables, written into buffers they own.
//
// The intermediate results (sinusoidal embeddings, the hidden layer and the
// output of the time MLP) live in one file-scope __device__ array of fixed
// size; the timestep grid travels by value in the kernel parameters.  Every call on a device shares it: calls whose work
// overlaps on the GPU (different streams, no ordering between them) race on
// it and must be serialised by the caller.  Each call overwrites every element
// it later reads, so nothing has to start at zero.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <mutex>

#include "internal.h"
#include "launch.cuh"
#include "pae.h"

namespace pae {

void set_create_error(const char* msg);  // pae_api.cu: message for pae_last_error(NULL)

namespace {

constexpr int kStaticMaxSteps = 64;     // largest K
constexpr int kStaticMaxWidth = 2048;   // largest width D
constexpr int kKc = 16;                 // timesteps per pass of the batched GEMV

// [ emb: K*D | z: K*D | c: K*D ] floats: 1.5 MB at the maximum sizes.
constexpr size_t kScratchFloats = 3 * (size_t)kStaticMaxSteps * kStaticMaxWidth;
__device__ __align__(256) float g_static_scratch[kScratchFloats];

// The timestep grid travels by value in the kernel parameters.
struct Grid {
  double t[kStaticMaxSteps + 1];
};

// Device address of g_static_scratch, looked up once per device (host code may
// not use the symbol itself: its host-side name is only a stand-in).
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
float* g_scratch_addr[kMaxDevices] = {};

template <typename TW>
__global__ void k_static_gemv(const TW* __restrict__ W, const TW* __restrict__ b, const float* __restrict__ in,
                              int K, int R, int D, int swish_out, float* __restrict__ out, size_t out_stride);

// Set-up, once per device with that device current: the scratch address and
// the kernels' shared-memory opt-in.
cudaError_t scratch_address(int dev, float** out) {
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return e;
    const int smem = (int)(kKc * kStaticMaxWidth * sizeof(float));
    e = cudaFuncSetAttribute(k_static_gemv<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(k_static_gemv<bf16>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = static_cast<float*>(p);
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

template <typename TW>
__device__ __forceinline__ float ldw(const TW* p);
template <>
__device__ __forceinline__ float ldw<float>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float ldw<bf16>(const bf16* p) { return bf2f(*p); }

// e_k = [sin(2 pi t_k / p_i), cos(2 pi t_k / p_i)], p_i geometric from 4e-3
// to 4.0 over D/2 periods; dt_k = t_{k+1} - t_k.
__global__ void k_static_embed(const Grid g, int D, float* __restrict__ emb, float* __restrict__ dt) {
  const double* t = g.t;
  const int k = blockIdx.x;
  const int half = D / 2;
  for (int i = threadIdx.x; i < half; i += blockDim.x) {
    const double frac = half > 1 ? (double)i / (double)(half - 1) : 0.0;
    const double period = 4e-3 * pow(4.0 / 4e-3, frac);
    const double ang = 2.0 * 3.141592653589793238 * t[k] / period;
    emb[(size_t)k * D + i] = (float)sin(ang);
    emb[(size_t)k * D + half + i] = (float)cos(ang);
  }
  if (threadIdx.x == 0) dt[k] = (float)(t[k + 1] - t[k]);
}

// out[k * out_stride + r] = act(W[r] . in[k] + b[r]) for k < K, r < R; one
// warp per row, up to kKc timesteps per pass staged in shared memory.
template <typename TW>
__global__ void k_static_gemv(const TW* __restrict__ W, const TW* __restrict__ b, const float* __restrict__ in,
                              int K, int R, int D, int swish_out, float* __restrict__ out, size_t out_stride) {
  extern __shared__ float xs[];  // [kKc][D]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int k0 = 0; k0 < K; k0 += kKc) {
    const int kc = min(kKc, K - k0);
    __syncthreads();
    for (int i = threadIdx.x; i < kc * D; i += blockDim.x) xs[i] = in[(size_t)k0 * D + i];
    __syncthreads();
    for (int r = blockIdx.x * nw + warp; r < R; r += gridDim.x * nw) {
      float acc[kKc];
#pragma unroll
      for (int j = 0; j < kKc; ++j) acc[j] = 0.f;
      const TW* wr = W + (size_t)r * D;
      for (int i = lane; i < D; i += 32) {
        const float w = ldw(wr + i);
#pragma unroll
        for (int j = 0; j < kKc; ++j)
          if (j < kc) acc[j] = fmaf(w, xs[j * D + i], acc[j]);
      }
      const float bias = ldw(b + r);
#pragma unroll
      for (int j = 0; j < kKc; ++j) {
        if (j < kc) {
          float v = warp_sum(acc[j]) + bias;
          if (swish_out) v = swishf(v);
          if (lane == 0) out[(size_t)(k0 + j) * out_stride + r] = v;
        }
      }
    }
  }
}

template <typename TW>
cudaError_t gemv(const void* W, const void* b, const float* in, int K, int R, int D, int swish_out, float* out,
                 size_t out_stride, cudaStream_t st) {
  const int threads = 256, wpb = threads / 32;
  int blocks = (R + wpb - 1) / wpb;
  if (blocks > 148 * 16) blocks = 148 * 16;
  const size_t smem = (size_t)kKc * D * sizeof(float);
  k_static_gemv<TW><<<blocks, threads, smem, st>>>(static_cast<const TW*>(W), static_cast<const TW*>(b), in, K, R, D,
                                                   swish_out, out, out_stride);
  return cudaGetLastError();
}

pae_status fail_static(pae_status st, const char* msg) {
  set_create_error(msg);
  return st;
}

}  // namespace
}  // namespace pae

using namespace pae;

extern "C" pae_status pae_precompute_tables_static(int layers, int width, int dtype, const pae_weights* w,
                                                   const double* t, int K, float* tables, float* dt,
                                                   pae_stream stream) {
  if (!w || !t || !tables || !dt)
    return fail_static(PAE_ERR_ARG, "pae_precompute_tables_static: a pointer argument is NULL");
  if (!w->w_t1 || !w->b_t1 || !w->w_t2 || !w->b_t2 || !w->w_mod || !w->b_mod || !w->w_modf || !w->b_modf)
    return fail_static(PAE_ERR_ARG, "pae_precompute_tables_static: a time-MLP or modulation weight is NULL");
  if (layers < 1 || width < 2 || width % 2 != 0)
    return fail_static(PAE_ERR_ARG, "pae_precompute_tables_static: layers must be >= 1 and width even");
  if (dtype != PAE_FP32 && dtype != PAE_BF16 && dtype != PAE_W4A16)
    return fail_static(PAE_ERR_ARG, "pae_precompute_tables_static: unknown dtype");
  if (K < 1 || K > kStaticMaxSteps)
    return fail_static(PAE_ERR_ARG, "pae_precompute_tables_static: K must be in [1, 64] (fixed scratch size)");
  if (width > kStaticMaxWidth)
    return fail_static(PAE_ERR_ARG, "pae_precompute_tables_static: width must be at most 2048 (fixed scratch size)");
  const double dir = t[1] - t[0];
  for (int k = 0; k < K; ++k)
    if (!((t[k + 1] - t[k]) * dir > 0.0))
      return fail_static(PAE_ERR_ARG, "pae_precompute_tables_static: t must be strictly monotone");

  // An error left pending by earlier, unrelated work would otherwise surface
  // from the launch checks below as if this call had caused it.
  cudaError_t e = cudaPeekAtLastError();
  if (e != cudaSuccess) {
    char msg[256];
    snprintf(msg, sizeof msg, "pae_precompute_tables_static: a CUDA error from earlier work is pending (%s)",
             cudaGetErrorString(e));
    return fail_static(PAE_ERR_CUDA, msg);
  }
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess)
    return fail_static(PAE_ERR_CUDA, "pae_precompute_tables_static: cudaGetDevice failed");
  if (dev < 0 || dev >= kMaxDevices)
    return fail_static(PAE_ERR_UNSUPPORTED, "pae_precompute_tables_static: device ordinals of 64 and above are "
                                            "not supported (per-device address cache)");
  float* scratch = nullptr;
  if ((e = scratch_address(dev, &scratch)) != cudaSuccess)
    return fail_static(PAE_ERR_CUDA, "pae_precompute_tables_static: cudaGetSymbolAddress failed");

  const int D = width;
  const size_t kd = (size_t)kStaticMaxSteps * kStaticMaxWidth;
  Grid grid{};
  for (int k = 0; k <= K; ++k) grid.t[k] = t[k];
  float* emb = scratch;
  float* z = emb + kd;
  float* c = z + kd;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool bf = dtype != PAE_FP32;
  const int mod_rows = layers * 2 * 3 * D;
  const size_t rows = (size_t)mod_rows + 2 * (size_t)D;  // per-step table length

  k_static_embed<<<K, 256, 0, st>>>(grid, D, emb, dt);
  e = cudaGetLastError();
  if (e == cudaSuccess)
    e = bf ? gemv<bf16>(w->w_t1, w->b_t1, emb, K, D, D, 1, z, D, st) : gemv<float>(w->w_t1, w->b_t1, emb, K, D, D, 1, z, D, st);
  if (e == cudaSuccess)
    e = bf ? gemv<bf16>(w->w_t2, w->b_t2, z, K, D, D, 1, c, D, st) : gemv<float>(w->w_t2, w->b_t2, z, K, D, D, 1, c, D, st);
  if (e == cudaSuccess)
    e = bf ? gemv<bf16>(w->w_mod, w->b_mod, c, K, mod_rows, D, 0, tables, rows, st)
           : gemv<float>(w->w_mod, w->b_mod, c, K, mod_rows, D, 0, tables, rows, st);
  if (e == cudaSuccess)
    e = bf ? gemv<bf16>(w->w_modf, w->b_modf, c, K, 2 * D, D, 0, tables + mod_rows, rows, st)
           : gemv<float>(w->w_modf, w->b_modf, c, K, 2 * D, D, 0, tables + mod_rows, rows, st);
  if (e != cudaSuccess) {
    set_create_error(cudaGetErrorString(e));
    return PAE_ERR_CUDA;
  }
  return PAE_OK;
}
