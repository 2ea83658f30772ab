// CUDA-core kernels of the fp32 mode: a tiled fp32 projection GEMM with the
// shared epilogues, and attention over [cached prefix | action keys].
#include <math.h>

#include "epilogue.cuh"

namespace pae {

namespace {

constexpr int BM = 32, BN = 64, BK = 32;

// out[m][f] = sum_k X[m][k] W[row(f)][k] with the epilogue e.  256 threads,
// each 2 tokens x 4 features (x 2 for GeGLU).
template <int NA>
__global__ void __launch_bounds__(256) k_gemm_f32(const Shape s, const float* __restrict__ X,
                                                  const float* __restrict__ W, int N, int K, const EpiArgs e) {
  __shared__ float xs[BK][BM + 1];
  __shared__ float ws[NA][BK][BN + 1];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int m0 = blockIdx.y * BM, f0 = blockIdx.x * BN;
  float acc[NA][2][4];
#pragma unroll
  for (int a = 0; a < NA; ++a)
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[a][i][j] = 0.f;

  for (int k0 = 0; k0 < K; k0 += BK) {
    for (int i = tid; i < BM * BK; i += 256) {
      const int mm = i / BK, kk = i - mm * BK;
      const int m = m0 + mm, k = k0 + kk;
      xs[kk][mm] = (m < e.M && k < K) ? X[(size_t)m * K + k] : 0.f;
    }
    for (int i = tid; i < NA * BN * BK; i += 256) {
      const int a = i / (BN * BK), r = i - a * BN * BK;
      const int nn = r / BK, kk = r - nn * BK;
      const int f = f0 + nn, k = k0 + kk;
      float v = 0.f;
      if (f < N && k < K) {
        const int row = NA == 2 ? gate_row(f) + a * 128 : f;
        v = W[(size_t)row * K + k];
      }
      ws[a][kk][nn] = v;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < BK; ++kk) {
      const float x0 = xs[kk][ty * 2], x1 = xs[kk][ty * 2 + 1];
#pragma unroll
      for (int a = 0; a < NA; ++a)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float w = ws[a][kk][tx * 4 + j];
          acc[a][0][j] = fmaf(x0, w, acc[a][0][j]);
          acc[a][1][j] = fmaf(x1, w, acc[a][1][j]);
        }
    }
    __syncthreads();
  }
  // q/k with rotation and the prefix keys/values go pair by pair: a thread's
  // four features are two stored pairs (f0 and 4 tx are even)
  const bool pairs = e.epi == EPI_PREFIX || (e.epi == EPI_QKV && e.rope_cs);
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int m = m0 + ty * 2 + i;
    if (m >= e.M) continue;
    if (pairs) {
#pragma unroll
      for (int j = 0; j < 4; j += 2) {
        const int f = f0 + tx * 4 + j;
        if (f >= N) continue;
        if (e.epi == EPI_PREFIX)
          epi_prefix_pair<float>(s, e, m, f, acc[0][i][j], acc[0][i][j + 1]);
        else
          epi_qkv_pair<float>(s, e, m, f, acc[0][i][j], acc[0][i][j + 1]);
      }
      continue;
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int f = f0 + tx * 4 + j;
      if (f >= N) continue;
      epi_apply<float>(s, e, m, f, acc[0][i][j], NA == 2 ? acc[NA - 1][i][j] : 0.f);
    }
  }
}

constexpr int MAXG = 16;

// One CTA per (request b, KV head g, action token i): the G query heads of
// the group share each key and value read.  s = q.k / sqrt(d) over keys
// [0, lens[b] + H) (prefix then this step's action keys); p = softmax(s);
// o = p . v.
template <typename TA>
__global__ void __launch_bounds__(256) k_attn_simple(const Shape s, const TA* __restrict__ q,
                                                     const TA* __restrict__ kc, const TA* __restrict__ vc,
                                                     const int* __restrict__ lens, int layer,
                                                     TA* __restrict__ o) {
  extern __shared__ float sm[];
  const int G = s.G, d = s.d;
  float* qs = sm;              // [G][d]
  float* sc = qs + G * d;      // [G][Ptot]
  const int b = blockIdx.x / s.Hkv, g = blockIdx.x - b * s.Hkv, i = blockIdx.y;
  const int n = lens[b] + s.H;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  for (int t = tid; t < G * d; t += blockDim.x) {
    const int hl = t / d, j = t - hl * d;
    const int hq = g * G + hl;
    qs[t] = ld_act<TA>(q + ((size_t)(b * s.Hq + hq) * s.H + i) * d + j);
  }
  __syncthreads();
  const size_t slot = ((size_t)(layer * s.Bmax + b) * s.Hkv + g) * s.Ptot;
  const float scale = rsqrtf((float)d);
  for (int key = warp; key < n; key += nw) {
    const TA* kr = kc + (slot + key) * d;
    float part[MAXG];
#pragma unroll
    for (int hl = 0; hl < MAXG; ++hl) part[hl] = 0.f;
    for (int j = lane; j < d; j += 32) {
      const float kv = ld_act<TA>(kr + j);
#pragma unroll
      for (int hl = 0; hl < MAXG; ++hl)
        if (hl < G) part[hl] = fmaf(qs[hl * d + j], kv, part[hl]);
    }
#pragma unroll
    for (int hl = 0; hl < MAXG; ++hl)
      if (hl < G) {
        const float v = warp_sum(part[hl]);
        if (lane == 0) sc[hl * s.Ptot + key] = v * scale;
      }
  }
  __syncthreads();
  for (int hl = warp; hl < G; hl += nw) {
    float* row = sc + hl * s.Ptot;
    float mx = -INFINITY;
    for (int k = lane; k < n; k += 32) mx = fmaxf(mx, row[k]);
    mx = warp_max(mx);
    float sum = 0.f;
    for (int k = lane; k < n; k += 32) {
      const float p = expf(row[k] - mx);
      row[k] = p;
      sum += p;
    }
    sum = warp_sum(sum);
    const float inv = 1.f / sum;
    for (int k = lane; k < n; k += 32) row[k] *= inv;
  }
  __syncthreads();
  const int m = b * s.H + i;
  for (int j = tid; j < d; j += blockDim.x) {
    float acc[MAXG];
#pragma unroll
    for (int hl = 0; hl < MAXG; ++hl) acc[hl] = 0.f;
    for (int k = 0; k < n; ++k) {
      const float v = ld_act<TA>(vc + (slot + k) * d + j);
#pragma unroll
      for (int hl = 0; hl < MAXG; ++hl)
        if (hl < G) acc[hl] = fmaf(sc[hl * s.Ptot + k], v, acc[hl]);
    }
#pragma unroll
    for (int hl = 0; hl < MAXG; ++hl)
      if (hl < G) st_act<TA>(o + (size_t)m * s.attn_dim + (g * G + hl) * d + j, acc[hl]);
  }
}

}  // namespace

void launch_gemm_simple(const Shape& s, const float* X, const float* W, int N, int K, const EpiArgs& e,
                        cudaStream_t st) {
  dim3 grid((N + BN - 1) / BN, (e.M + BM - 1) / BM);
  if (e.epi == EPI_GEGLU)
    k_gemm_f32<2><<<grid, 256, 0, st>>>(s, X, W, N, K, e);
  else
    k_gemm_f32<1><<<grid, 256, 0, st>>>(s, X, W, N, K, e);
}

void launch_attention_simple(const Shape& s, int act_bf16, const void* q, const void* kc, const void* vc,
                             const int* lens, int layer, void* o, int B, cudaStream_t st) {
  dim3 grid(B * s.Hkv, s.H);
  const size_t smem = (size_t)s.G * (s.d + s.Ptot) * sizeof(float);
  if (act_bf16) {
    if (smem > 48 * 1024)
      cudaFuncSetAttribute(k_attn_simple<bf16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k_attn_simple<bf16><<<grid, 256, smem, st>>>(s, static_cast<const bf16*>(q), static_cast<const bf16*>(kc),
                                                 static_cast<const bf16*>(vc), lens, layer, static_cast<bf16*>(o));
  } else {
    if (smem > 48 * 1024)
      cudaFuncSetAttribute(k_attn_simple<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k_attn_simple<float><<<grid, 256, smem, st>>>(s, static_cast<const float*>(q), static_cast<const float*>(kc),
                                                  static_cast<const float*>(vc), lens, layer,
                                                  static_cast<float*>(o));
  }
}

}  // namespace pae
