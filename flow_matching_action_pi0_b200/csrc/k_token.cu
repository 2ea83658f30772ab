// Token-local kernels of the denoise loop.
//
// k_transition joins two consecutive Euler steps, since everything between
// them is local to one action token:
//   (end of step k)   y = adaRMSNorm(h; final scale/shift), v = y W_out^T + b_out,
//                     x += dt_k v                                  (Euler update)
//   (start of k+1)    h = x W_in^T + b_in,
//                     y = adaRMSNorm(h; layer-0 attention scale/shift)
// adaRMSNorm(h) = h / sqrt(mean(h^2) + eps) * (1 + scale) + shift (no learned gain).
// Reductions use a fixed tree, so results are bitwise reproducible.
#include "internal.h"
#include "launch.cuh"

namespace pae {

namespace {

template <typename TW>
__device__ __forceinline__ float ldw(const TW* p);
template <>
__device__ __forceinline__ float ldw<float>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float ldw<bf16>(const bf16* p) { return bf2f(*p); }

// One CTA per token.  w_in is stored transposed ([A][D]) so that the D outputs
// read it coalesced.
template <typename TW, typename TA>
__global__ void __launch_bounds__(256) k_transition(const Shape s, const TransitionArgs a) {
  extern __shared__ float sm[];
  float* hs = sm;             // [D]
  float* xs = hs + s.D;       // [A]
  float* red = xs + s.A;      // [32]
  const int m = blockIdx.x;
  const int D = s.D, A = s.A;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  const float* xsrc = a.x_src + (size_t)m * A;
  float* xdst = a.x_dst + (size_t)m * A;
  pdl_wait();
  pdl_launch_dependents();

  if (a.tab_out) {
    const float* hrow = a.h + (size_t)m * D;
    float ss = 0.f;
    for (int j = tid; j < D; j += blockDim.x) {
      const float v = hrow[j];
      hs[j] = v;
      ss = fmaf(v, v, ss);
    }
    ss = block_sum(ss, red);
    const float r = rsqrtf(ss / (float)D + s.eps);
    const float* sc = a.tab_out + final_offset(s, 0);
    const float* sh = a.tab_out + final_offset(s, 1);
    __syncthreads();
    for (int j = tid; j < D; j += blockDim.x) hs[j] = hs[j] * r * (1.f + sc[j]) + sh[j];
    __syncthreads();
    const TW* wout = static_cast<const TW*>(a.w_out);
    const TW* bout = static_cast<const TW*>(a.b_out);
    const float dtk = a.dt[a.k_out];
    for (int o = warp; o < A; o += nw) {
      float acc = 0.f;
      const TW* wr = wout + (size_t)o * D;
      for (int j = lane; j < D; j += 32) acc = fmaf(hs[j], ldw(wr + j), acc);
      acc = warp_sum(acc);
      if (lane == 0) {
        const float v = acc + ldw(bout + o);
        const float xn = xsrc[o] + dtk * v;
        xdst[o] = xn;
        xs[o] = xn;
      }
    }
    __syncthreads();
  } else {
    for (int o = tid; o < A; o += blockDim.x) xs[o] = xsrc[o];
    __syncthreads();
  }

  if (a.tab_in) {
    const TW* winT = static_cast<const TW*>(a.w_in);  // [A][D]
    const TW* bin = static_cast<const TW*>(a.b_in);
    float* hrow = a.h + (size_t)m * D;
    float ss = 0.f;
    for (int j = tid; j < D; j += blockDim.x) {
      float acc = ldw(bin + j);
      for (int o = 0; o < A; ++o) acc = fmaf(xs[o], ldw(winT + (size_t)o * D + j), acc);
      hs[j] = acc;
      hrow[j] = acc;
      ss = fmaf(acc, acc, ss);
    }
    ss = block_sum(ss, red);
    const float r = rsqrtf(ss / (float)D + s.eps);
    const float* sc = a.tab_in + mod_offset(s, 0, 0, 0);
    const float* sh = a.tab_in + mod_offset(s, 0, 0, 1);
    TA* yrow = static_cast<TA*>(a.y) + (size_t)m * D;
    for (int j = tid; j < D; j += blockDim.x) st_act<TA>(yrow + j, hs[j] * r * (1.f + sc[j]) + sh[j]);
  }
}

// One warp per token.
template <typename TA>
__global__ void __launch_bounds__(256) k_norm(const Shape s, const float* __restrict__ h, TA* __restrict__ y,
                                              const float* __restrict__ scale, const float* __restrict__ shift,
                                              int M) {
  const int lane = threadIdx.x & 31;
  const int m = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  pdl_wait();
  pdl_launch_dependents();
  if (m >= M) return;
  const int D = s.D;
  const float* hr = h + (size_t)m * D;
  float ss = 0.f;
  for (int j = lane; j < D; j += 32) ss = fmaf(hr[j], hr[j], ss);
  ss = warp_sum(ss);
  const float r = rsqrtf(ss / (float)D + s.eps);
  TA* yr = y + (size_t)m * D;
  for (int j = lane; j < D; j += 32) st_act<TA>(yr + j, hr[j] * r * (1.f + scale[j]) + shift[j]);
}

}  // namespace

cudaError_t launch_transition(const Shape& s, int act_bf16, const TransitionArgs& a, bool pdl, cudaStream_t st) {
  const size_t smem = (size_t)(s.D + s.A + 32) * sizeof(float);
  if (act_bf16) return launch_ex(k_transition<bf16, bf16>, dim3(a.M), dim3(256), smem, st, 1, pdl, s, a);
  return launch_ex(k_transition<float, float>, dim3(a.M), dim3(256), smem, st, 1, pdl, s, a);
}

cudaError_t launch_norm(const Shape& s, int act_bf16, const float* h, void* y, const float* scale, const float* shift,
                        int M, bool pdl, cudaStream_t st) {
  const int blocks = (M + 7) / 8;
  if (act_bf16)
    return launch_ex(k_norm<bf16>, dim3(blocks), dim3(256), 0, st, 1, pdl, s, h, static_cast<bf16*>(y), scale, shift,
                     M);
  return launch_ex(k_norm<float>, dim3(blocks), dim3(256), 0, st, 1, pdl, s, h, static_cast<float*>(y), scale, shift,
                   M);
}

}  // namespace pae
