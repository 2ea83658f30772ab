// Token-local kernels of the denoise loop.
//
// k_transition joins two consecutive Euler steps, since everything between
// them is local to one action token:
//   (end of step k)   y = adaRMSNorm(h; final scale/shift), v = y W_out^T + b_out,
//                     x += dt_k v                                  (Euler update)
//   (start of k+1)    h = x W_in^T + b_in,
//                     y = adaRMSNorm(h; layer-0 attention scale/shift)
// adaRMSNorm(h) = h / sqrt(mean(h^2) + eps) * (1 + scale) + shift (no learned gain).
// These kernels are latency-bound (tens of KB per token), so every thread
// issues all of its 16-byte loads before it uses any of them.  Reductions use
// a fixed tree, so results are bitwise reproducible.
#include "internal.h"
#include "launch.cuh"

namespace pae {

namespace {

// 8 consecutive weights as floats (16-byte loads for bf16, 2 x 16 for fp32).
__device__ __forceinline__ void load8(const bf16* p, float* w) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t q[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    w[2 * i] = __uint_as_float(q[i] << 16);
    w[2 * i + 1] = __uint_as_float(q[i] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void load8(const float* p, float* w) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
  w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
}
// 4 consecutive values as floats.
__device__ __forceinline__ void load4(const bf16* p, float* w) {
  const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
  w[0] = __uint_as_float(u.x << 16);
  w[1] = __uint_as_float(u.x & 0xFFFF0000u);
  w[2] = __uint_as_float(u.y << 16);
  w[3] = __uint_as_float(u.y & 0xFFFF0000u);
}
__device__ __forceinline__ void load4(const float* p, float* w) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
}
__device__ __forceinline__ void store4(bf16* p, const float* v) {
  const uint32_t a = (uint32_t)__bfloat16_as_ushort(f2bf(v[0])) | ((uint32_t)__bfloat16_as_ushort(f2bf(v[1])) << 16);
  const uint32_t b = (uint32_t)__bfloat16_as_ushort(f2bf(v[2])) | ((uint32_t)__bfloat16_as_ushort(f2bf(v[3])) << 16);
  *reinterpret_cast<uint2*>(p) = make_uint2(a, b);
}
__device__ __forceinline__ void store4(float* p, const float* v) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}

// One CTA (256 threads) per token.  w_in is stored transposed ([A][D]).
// Requires D % 8 == 0 (16-byte weight loads).
template <typename TW, typename TA>
__global__ void __launch_bounds__(256) k_transition(const Shape s, const TransitionArgs a) {
  GTRACE_BEGIN();
  extern __shared__ float sm[];
  float* hs = sm;             // [D]
  float* xs = hs + s.D;       // [A]
  float* red = xs + s.A;      // [32]
  const int m = blockIdx.x;
  const int D = s.D, A = s.A;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  const float* xsrc = a.x_src + (size_t)m * A;
  float* xdst = a.x_dst + (size_t)m * A;
  // This kernel holds no TMEM, so its successor (a projection, which only
  // streams weights before its own wait) may be scheduled at once.
  pdl_launch_dependents();
  pdl_wait();
  GTRACE_WAITED();

  if (a.tab_out) {
    const float* hrow = a.h + (size_t)m * D;
    const float* sc = a.tab_out + final_offset(s, 0);
    const float* sh = a.tab_out + final_offset(s, 1);
    float ss = 0.f;
    for (int j = 4 * tid; j < D; j += 4 * blockDim.x) {
      const float4 v = *reinterpret_cast<const float4*>(hrow + j);
      *reinterpret_cast<float4*>(hs + j) = v;
      ss = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, ss))));
    }
    ss = block_sum(ss, red);
    const float r = rsqrtf(ss / (float)D + s.eps);
    for (int j = 4 * tid; j < D; j += 4 * blockDim.x) {
      float4 v = *reinterpret_cast<const float4*>(hs + j);
      const float4 c = *reinterpret_cast<const float4*>(sc + j);
      const float4 d = *reinterpret_cast<const float4*>(sh + j);
      v.x = v.x * r * (1.f + c.x) + d.x;
      v.y = v.y * r * (1.f + c.y) + d.y;
      v.z = v.z * r * (1.f + c.z) + d.z;
      v.w = v.w * r * (1.f + c.w) + d.w;
      *reinterpret_cast<float4*>(hs + j) = v;
    }
    __syncthreads();
    // v = y W_out^T + b_out: warp w takes outputs w, w+8, ...; each lane 8
    // consecutive inputs per 256-wide chunk, all loads issued up front.
    const TW* wout = static_cast<const TW*>(a.w_out);
    const TW* bout = static_cast<const TW*>(a.b_out);
    const float dtk = a.dt[a.k_out];
    for (int o0 = warp; o0 < A; o0 += 4 * nw) {
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      for (int j0 = 8 * lane; j0 < D; j0 += 256) {
        float w[4][8];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int o = o0 + u * nw;
          if (o < A) load8(wout + (size_t)o * D + j0, w[u]);
        }
        const float4 y0 = *reinterpret_cast<const float4*>(hs + j0);
        const float4 y1 = *reinterpret_cast<const float4*>(hs + j0 + 4);
        const float yv[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (o0 + u * nw < A)
#pragma unroll
            for (int t = 0; t < 8; ++t) acc[u] = fmaf(yv[t], w[u][t], acc[u]);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int o = o0 + u * nw;
        const float v = warp_sum(acc[u]);
        if (lane == 0 && o < A) {
          float bo;
          if constexpr (sizeof(TW) == 2) bo = bf2f(bout[o]); else bo = bout[o];
          const float xn = xsrc[o] + dtk * (v + bo);
          xdst[o] = xn;
          xs[o] = xn;
        }
      }
    }
    __syncthreads();
  } else {
    for (int o = tid; o < A; o += blockDim.x) xs[o] = xsrc[o];
    __syncthreads();
  }

  if (a.tab_in) {
    // h = x W_in^T + b_in: thread owns 4 consecutive features per 1024-wide chunk.
    const TW* winT = static_cast<const TW*>(a.w_in);  // [A][D]
    const TW* bin = static_cast<const TW*>(a.b_in);
    float* hrow = a.h + (size_t)m * D;
    float ss = 0.f;
    for (int j = 4 * tid; j < D; j += 4 * blockDim.x) {
      float acc[4];
      load4(bin + j, acc);
      for (int o0 = 0; o0 < A; o0 += 16) {
        float w[16][4];
#pragma unroll
        for (int u = 0; u < 16; ++u)
          if (o0 + u < A) load4(winT + (size_t)(o0 + u) * D + j, w[u]);
#pragma unroll
        for (int u = 0; u < 16; ++u)
          if (o0 + u < A) {
            const float xv = xs[o0 + u];
#pragma unroll
            for (int t = 0; t < 4; ++t) acc[t] = fmaf(xv, w[u][t], acc[t]);
          }
      }
      *reinterpret_cast<float4*>(hs + j) = make_float4(acc[0], acc[1], acc[2], acc[3]);
      *reinterpret_cast<float4*>(hrow + j) = make_float4(acc[0], acc[1], acc[2], acc[3]);
      ss = fmaf(acc[0], acc[0], fmaf(acc[1], acc[1], fmaf(acc[2], acc[2], fmaf(acc[3], acc[3], ss))));
    }
    ss = block_sum(ss, red);
    if (a.ss_out && tid == 0) a.ss_out[m] = ss;  // slot 0 for a projection that normalises in-kernel
    // factored: the projection applies rstd and the shift term itself
    const float r = a.y_factored ? 1.f : rsqrtf(ss / (float)D + s.eps);
    const float* sc = a.tab_in + mod_offset(s, 0, 0, 0);
    const float* sh = a.tab_in + mod_offset(s, 0, 0, 1);
    TA* yrow = static_cast<TA*>(a.y) + (size_t)m * D;
    for (int j = 4 * tid; j < D; j += 4 * blockDim.x) {
      const float4 v = *reinterpret_cast<const float4*>(hs + j);
      const float4 c = *reinterpret_cast<const float4*>(sc + j);
      const float4 d = a.y_factored ? make_float4(0.f, 0.f, 0.f, 0.f) : *reinterpret_cast<const float4*>(sh + j);
      const float o[4] = {v.x * r * (1.f + c.x) + d.x, v.y * r * (1.f + c.y) + d.y, v.z * r * (1.f + c.z) + d.z,
                          v.w * r * (1.f + c.w) + d.w};
      store4(yrow + j, o);
    }
  }
  GTRACE_END(6);
}

// One warp per token; the row stays in registers (NV float4 per lane).
template <typename TA, int NV>
__global__ void __launch_bounds__(256) k_norm(const Shape s, const float* __restrict__ h, TA* __restrict__ y,
                                              const float* __restrict__ scale, const float* __restrict__ shift,
                                              int M) {
  GTRACE_BEGIN();
  const int lane = threadIdx.x & 31;
  const int m = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int D = s.D;
  // The modulation rows are built before the loop, not by the previous
  // kernel: read them before waiting for it.
  float4 cs[NV], ds[NV];
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int j = 4 * (lane + 32 * i);
    if (j < D && m < M) {
      cs[i] = __ldg(reinterpret_cast<const float4*>(scale + j));
      ds[i] = __ldg(reinterpret_cast<const float4*>(shift + j));
    }
  }
  // No TMEM or other resource is taken after this point, so the successor (a
  // projection) is let in before the wait: its CTAs become resident while the
  // projection before this kernel still runs and stream their weights early.
  pdl_launch_dependents();
  pdl_wait();
  GTRACE_WAITED();
  if (m >= M) return;
  const float* hr = h + (size_t)m * D;
  float4 v[NV];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int j = 4 * (lane + 32 * i);
    v[i] = j < D ? *reinterpret_cast<const float4*>(hr + j) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int i = 0; i < NV; ++i) ss = fmaf(v[i].x, v[i].x, fmaf(v[i].y, v[i].y, fmaf(v[i].z, v[i].z, fmaf(v[i].w, v[i].w, ss))));
  ss = warp_sum(ss);
  const float r = rsqrtf(ss / (float)D + s.eps);
  TA* yr = y + (size_t)m * D;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int j = 4 * (lane + 32 * i);
    if (j < D) {
      const float4 c = cs[i];
      const float4 d = ds[i];
      const float o[4] = {v[i].x * r * (1.f + c.x) + d.x, v[i].y * r * (1.f + c.y) + d.y,
                          v[i].z * r * (1.f + c.z) + d.z, v[i].w * r * (1.f + c.w) + d.w};
      store4(yr + j, o);
    }
  }
  GTRACE_END(5);
}

template <typename TA>
cudaError_t norm_dispatch(const Shape& s, const float* h, TA* y, const float* scale, const float* shift, int M,
                          bool pdl, cudaStream_t st) {
  const dim3 grid((M + 7) / 8), block(256);
  const int nv = (s.D + 127) / 128;
  if (nv <= 2) return launch_ex(k_norm<TA, 2>, grid, block, 0, st, 1, pdl, s, h, y, scale, shift, M);
  if (nv <= 4) return launch_ex(k_norm<TA, 4>, grid, block, 0, st, 1, pdl, s, h, y, scale, shift, M);
  if (nv <= 8) return launch_ex(k_norm<TA, 8>, grid, block, 0, st, 1, pdl, s, h, y, scale, shift, M);
  return launch_ex(k_norm<TA, 16>, grid, block, 0, st, 1, pdl, s, h, y, scale, shift, M);
}

// Prefix production, step 1: y = h / sqrt(mean(h^2) + eps) per prefix token
// (a plain RMSNorm; one warp per token, the sum of squares in fp32 in a fixed
// lane order).
template <typename TA>
__global__ void __launch_bounds__(256) k_prefix_norm(const TA* __restrict__ h, TA* __restrict__ y, int len, int Dp,
                                                     float eps) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m = blockIdx.x * 8 + warp;
  if (m >= len) return;
  const TA* hr = h + (size_t)m * Dp;
  float ss = 0.f;
  for (int j = lane; j < Dp; j += 32) {
    const float v = ld_act<TA>(hr + j);
    ss = fmaf(v, v, ss);
  }
  ss = warp_sum(ss);
  const float r = rsqrtf(ss / (float)Dp + eps);
  TA* yr = y + (size_t)m * Dp;
  for (int j = lane; j < Dp; j += 32) st_act<TA>(yr + j, ld_act<TA>(hr + j) * r);
}

}  // namespace

cudaError_t launch_prefix_norm(int act_bf16, const void* h, void* y, int len, int Dp, float eps, cudaStream_t st) {
  const dim3 grid((len + 7) / 8), block(256);
  if (act_bf16)
    k_prefix_norm<bf16><<<grid, block, 0, st>>>(static_cast<const bf16*>(h), static_cast<bf16*>(y), len, Dp, eps);
  else
    k_prefix_norm<float><<<grid, block, 0, st>>>(static_cast<const float*>(h), static_cast<float*>(y), len, Dp, eps);
  return cudaGetLastError();
}

cudaError_t launch_transition(const Shape& s, int act_bf16, const TransitionArgs& a, bool pdl, cudaStream_t st) {
  const size_t smem = (size_t)(s.D + s.A + 32) * sizeof(float);
  if (act_bf16) return launch_ex(k_transition<bf16, bf16>, dim3(a.M), dim3(256), smem, st, 1, pdl, s, a);
  return launch_ex(k_transition<float, float>, dim3(a.M), dim3(256), smem, st, 1, pdl, s, a);
}

cudaError_t launch_norm(const Shape& s, int act_bf16, const float* h, void* y, const float* scale, const float* shift,
                        int M, bool pdl, cudaStream_t st) {
  if (act_bf16) return norm_dispatch<bf16>(s, h, static_cast<bf16*>(y), scale, shift, M, pdl, st);
  return norm_dispatch<float>(s, h, static_cast<float*>(y), scale, shift, M, pdl, st);
}

}  // namespace pae

#ifdef PAE_GRAPH_TRACE
// Trace builds only: hand this file's kernels the launch-trace buffer.
extern "C" int pae_graph_trace_bind_token(void* buf, void* ctr, unsigned cap) {
  return (int)pae::gtrace_bind_tu(buf, ctr, cap);
}
#endif
