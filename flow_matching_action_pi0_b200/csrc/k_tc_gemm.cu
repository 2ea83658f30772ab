// Weight-streaming projection GEMM on the 5th-generation tensor cores.
//
//   out[m][f] = sum_k X[m][k] W[f][k]   followed by one of the epilogues
//   (q/k/v scatter, gated residual, GeGLU).
//
// The weights are the MMA's M side (128 rows per tile, or 2 x 128 for the
// interleaved gate/up tile) and the action tokens are its N side, so a chunk of
// 50 tokens costs one N=64 MMA per 16-wide K step instead of padding tokens to
// 128.  Per CTA:
//   warp 0 / lane 0  TMA producer: weight tile [128*NA][64] and token tile
//                    [tn][64] per stage, both 128-byte swizzled, into a ring
//   warp 1 / lane 0  MMA issuer: tcgen05.mma kind::f16 (bf16 in, fp32 in TMEM)
//   warps 0-3        epilogue: tcgen05.ld of the accumulator (thread = weight
//                    row = output feature, 16 token columns per load)
// Split-K: grid.y CTAs share one output tile; each writes its fp32 partial to a
// workspace, and the last CTA to arrive (atomic counter) sums the partials in
// split order and runs the epilogue.  No CTA waits for another, and the sum
// order is fixed, so results are bitwise reproducible.
#include "epilogue.cuh"

namespace pae {

namespace {

// Loads and MMAs always finish in bounded time; waits for them after an abort
// (draining) get this fixed bound instead of the short pipeline limit.
constexpr long long kDrainNs = 4000000000LL;

__host__ __device__ inline uint32_t tmem_cols_for(int n) {
  uint32_t c = 32;
  while ((int)c < n) c <<= 1;
  return c;
}

struct TcSmemLayout {
  uint32_t a_bytes, b_bytes, stage_bytes, bar_off, total;
};

__host__ __device__ inline TcSmemLayout tc_layout(int na, int tn, int stages) {
  TcSmemLayout L;
  L.a_bytes = (uint32_t)na * 128u * 128u;
  L.b_bytes = (uint32_t)tn * 128u;
  L.stage_bytes = L.a_bytes + L.b_bytes;
  L.bar_off = L.stage_bytes * (uint32_t)stages;
  L.total = L.bar_off + 256 + 1024;  // barriers + slack for 1024-byte alignment
  return L;
}

template <int NA>
__global__ void __launch_bounds__(128, 1)
    k_tc_gemm(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX, const Shape s,
              const TcPlan p, const TcGemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const TcSmemLayout L = tc_layout(NA, p.tn, p.stages);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bar_off);
  uint64_t* empty = full + p.stages;
  uint64_t* accf = empty + p.stages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);
  volatile int* s_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);  // [0] abort, [1] last

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntile = blockIdx.x, split = blockIdx.y, ttile = blockIdx.z;
  const int kps = a.K / p.splits;
  const int k0 = split * kps;
  const int nkb = kps / 64;
  const uint32_t ncols = tmem_cols_for(NA * p.tn);

  if (threadIdx.x == 0) {
    for (int i = 0; i < p.stages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(accf, 1);
    s_flag[0] = 0;
    s_flag[1] = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, ncols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- producer
    const uint64_t pol_w = policy_evict_first();  // weights: streamed once
    int issued = 0;
    for (int kb = 0; kb < nkb; ++kb) {
      const int st = kb % p.stages;
      if (kb >= p.stages) {
        if (!mbar_wait(&empty[st], ((kb / p.stages) & 1) ^ 1, a.err.wait_ns)) {
          s_flag[0] = 1;
          set_error(a.err, DEV_TIMEOUT);
          break;
        }
      }
      uint8_t* sa = smem + (size_t)st * L.stage_bytes;
      mbar_arrive_expect_tx(&full[st], L.stage_bytes);
      tma_load_2d_hint(sa, &tmW, k0 + kb * 64, a.w_row0 + ntile * 128 * NA, &full[st], pol_w);
      tma_load_2d(sa + L.a_bytes, &tmX, k0 + kb * 64, ttile * p.tn, &full[st]);
      issued = kb + 1;
    }
    // Loads still in flight must land before this CTA may exit.
    for (int kb = issued > p.stages ? issued - p.stages : 0; kb < issued; ++kb)
      if (!mbar_wait(&full[kb % p.stages], (kb / p.stages) & 1, kDrainNs)) set_error(a.err, DEV_TIMEOUT);
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------------- MMA
    const uint32_t idesc = idesc_bf16(128, p.tn);
    for (int kb = 0; kb < nkb; ++kb) {
      const int st = kb % p.stages;
      if (!mbar_wait(&full[st], (kb / p.stages) & 1, a.err.wait_ns)) {
        s_flag[0] = 1;
        set_error(a.err, DEV_TIMEOUT);
        break;
      }
      tc_fence_after();
      const uint32_t sa = smem_u32(smem + (size_t)st * L.stage_bytes);
      const uint32_t sb = sa + L.a_bytes;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t bdesc = sw128_desc(sb + kk * 32, 16, 1024);
#pragma unroll
        for (int na = 0; na < NA; ++na) {
          const uint64_t adesc = sw128_desc(sa + na * 16384 + kk * 32, 16, 1024);
          umma_bf16(tmem + na * p.tn, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
        }
      }
      umma_commit(&empty[st]);  // stage reusable once these MMAs have read it
    }
    umma_commit(accf);  // always issued, so the epilogue wait ends
  }
  __syncwarp();

  // ------------------------------------------------------------------ epilogue
  const bool acc_ok = mbar_wait(accf, 0, kDrainNs);
  if (!acc_ok) set_error(a.err, DEV_TIMEOUT);
  tc_fence_after();
  // CTA-uniform decision: the TMEM loads below are warp-collective.
  const bool ok = __syncthreads_and(acc_ok ? 1 : 0) != 0 && s_flag[0] == 0;

  const int row = warp * 32 + lane;
  const int f = ntile * 128 + row;
  const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
  const int mbase = ttile * p.tn;
  const EpiArgs& e = a.e;

  if (ok && p.splits == 1) {
    for (int c0 = 0; c0 < p.tn; c0 += 16) {
      float v0[16], v1[16];
      tmem_ld16(trow + c0, v0);
      if (NA == 2) tmem_ld16(trow + p.tn + c0, v1);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int m = mbase + c0 + j;
        if (m < e.M && f < a.N) epi_apply<bf16>(s, e, m, f, v0[j], NA == 2 ? v1[j] : 0.f);
      }
    }
  } else if (ok) {
    const size_t Mpad = (size_t)p.tok_tiles * p.tn;
    for (int c0 = 0; c0 < p.tn; c0 += 16) {
      float v0[16], v1[16];
      tmem_ld16(trow + c0, v0);
      if (NA == 2) tmem_ld16(trow + p.tn + c0, v1);
      tmem_ld_wait();
      if (f < a.N) {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const size_t m = mbase + c0 + j;
          a.partials[((size_t)(split * NA) * Mpad + m) * a.N + f] = v0[j];
          if (NA == 2) a.partials[((size_t)(split * NA + 1) * Mpad + m) * a.N + f] = v1[j];
        }
      }
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
      int* ctr = a.counters + ttile * gridDim.x + ntile;
      const int prev = atomicAdd(ctr, 1);
      const int last = (prev == p.splits - 1);
      s_flag[1] = last;
      if (last) *ctr = 0;  // every split has arrived: reset for the next launch
    }
    __syncthreads();
    if (s_flag[1]) {
      __threadfence();
      if (f < a.N) {
        for (int c = 0; c < p.tn; ++c) {
          const int m = mbase + c;
          if (m >= e.M) break;
          float s0 = 0.f, s1 = 0.f;
          for (int sp = 0; sp < p.splits; ++sp) {
            s0 += __ldcg(&a.partials[((size_t)(sp * NA) * Mpad + m) * a.N + f]);
            if (NA == 2) s1 += __ldcg(&a.partials[((size_t)(sp * NA + 1) * Mpad + m) * a.N + f]);
          }
          epi_apply<bf16>(s, e, m, f, s0, s1);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, ncols);
}

}  // namespace

size_t tc_gemm_smem_bytes(int na, const TcPlan& p) { return tc_layout(na, p.tn, p.stages).total; }

cudaError_t tc_gemm_init() {
  const int max_smem = 227 * 1024;
  cudaError_t e = cudaFuncSetAttribute(k_tc_gemm<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(k_tc_gemm<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
}

void launch_tc_gemm(const Shape& s, const CUtensorMap* tmW, const CUtensorMap* tmX, int na, const TcPlan& p,
                    const TcGemmArgs& a, cudaStream_t st) {
  const int ntiles = (a.N + 127) / 128;
  dim3 grid(ntiles, p.splits, p.tok_tiles);
  const size_t smem = tc_gemm_smem_bytes(na, p);
  if (na == 2)
    k_tc_gemm<2><<<grid, 128, smem, st>>>(*tmW, *tmX, s, p, a);
  else
    k_tc_gemm<1><<<grid, 128, smem, st>>>(*tmW, *tmX, s, p, a);
}

}  // namespace pae
