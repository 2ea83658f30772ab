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
// Split-K: the grid.y CTAs of one output tile form a thread-block cluster;
// their fp32 partials are reduced on chip through distributed shared memory,
// each CTA summing a 1/S slice of the rows over all ranks in rank order, so
// results are bitwise reproducible and no partial touches global memory.
// The weight loads of the first ring are issued before griddepcontrol.wait, so
// under programmatic dependent launch they overlap the previous kernel.
#include "epilogue.cuh"
#include "launch.cuh"

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
  volatile int* s_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);  // [0] abort

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
  // Only now, with its TMEM held, may this CTA let the next kernel's CTAs in:
  // a successor that took the TMEM first would wait on us forever.
  pdl_launch_dependents();

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- producer
    // Weight tiles do not depend on the previous kernel: the first ring's worth
    // is requested before waiting for it (programmatic dependent launch).
    // weights are streamed once per step when one token tile covers the batch;
    // otherwise the other token tiles re-read them from L2
    const uint64_t pol_w = p.tok_tiles == 1 ? policy_evict_first() : policy_evict_last();
    const int npre = nkb < p.stages ? nkb : p.stages;
    const int wrow = a.w_row0 + ntile * 128 * NA;
    for (int kb = 0; kb < npre; ++kb) {
      mbar_arrive_expect_tx(&full[kb], L.stage_bytes);
      tma_load_2d_hint(smem + (size_t)kb * L.stage_bytes, &tmW, k0 + kb * 64, wrow, &full[kb], pol_w);
    }
    pdl_wait();
    for (int kb = 0; kb < npre; ++kb)
      tma_load_2d(smem + (size_t)kb * L.stage_bytes + L.a_bytes, &tmX, k0 + kb * 64, ttile * p.tn, &full[kb]);
    int issued = npre;
    for (int kb = npre; kb < nkb; ++kb) {
      const int st = kb % p.stages;
      if (!mbar_wait(&empty[st], ((kb / p.stages) & 1) ^ 1, a.err.wait_ns)) {
        s_flag[0] = 1;
        set_error(a.err, DEV_TIMEOUT);
        break;
      }
      uint8_t* sa = smem + (size_t)st * L.stage_bytes;
      mbar_arrive_expect_tx(&full[st], L.stage_bytes);
      tma_load_2d_hint(sa, &tmW, k0 + kb * 64, wrow, &full[st], pol_w);
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
  pdl_wait();  // the epilogue reads the residual stream / slot lengths

  // ------------------------------------------------------------------ epilogue
  const bool acc_ok = mbar_wait(accf, 0, kDrainNs);
  if (!acc_ok) set_error(a.err, DEV_TIMEOUT);
  tc_fence_after();
  // CTA-uniform decision: the TMEM loads below are warp-collective.
  const bool ok = __syncthreads_and(acc_ok ? 1 : 0) != 0 && s_flag[0] == 0;

  const int row = warp * 32 + lane;
  const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
  const int mbase = ttile * p.tn;
  const EpiArgs& e = a.e;

  if (p.splits == 1) {
    const int f = ntile * 128 + row;
    if (ok) {
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
    }
  } else {
    // Split-K inside a cluster of p.splits CTAs: each parks its fp32 partial
    // in its own shared memory, token-major ([na][token][128 rows]), then CTA
    // rank r sums rows [r*R, r*R+R) over all ranks in rank order through
    // distributed shared memory and runs the epilogue on them.
    float* red = reinterpret_cast<float*>(smem);
    if (ok) {
      for (int c0 = 0; c0 < p.tn; c0 += 16) {
        float v0[16], v1[16];
        tmem_ld16(trow + c0, v0);
        if (NA == 2) tmem_ld16(trow + p.tn + c0, v1);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          red[(c0 + j) * 128 + row] = v0[j];
          if (NA == 2) red[(p.tn + c0 + j) * 128 + row] = v1[j];
        }
      }
    }
    cluster_sync();
    const int S = p.splits;
    const uint32_t rank = cluster_rank();
    const int R = 128 / S;
    const uint32_t red_base = smem_u32(red);
    const int any_ok = ok ? 1 : 0;
    if (any_ok) {
      for (int el = threadIdx.x; el < R * p.tn; el += 128) {
        const int rr = el % R, col = el / R;
        const int rw = (int)rank * R + rr;
        const int m = mbase + col, f = ntile * 128 + rw;
        const uint32_t off0 = (uint32_t)((col * 128 + rw) * 4);
        const uint32_t off1 = (uint32_t)(((p.tn + col) * 128 + rw) * 4);
        // issue every rank's load first (they pipeline), then sum in rank order
        float v0[16], v1[16];
#pragma unroll
        for (int q = 0; q < 16; ++q)
          if (q < S) {
            v0[q] = ld_cluster_f32(map_cluster(red_base + off0, (uint32_t)q));
            if (NA == 2) v1[q] = ld_cluster_f32(map_cluster(red_base + off1, (uint32_t)q));
          }
        float s0 = 0.f, s1 = 0.f;
#pragma unroll
        for (int q = 0; q < 16; ++q)
          if (q < S) {
            s0 += v0[q];
            if (NA == 2) s1 += v1[q];
          }
        if (m < e.M && f < a.N) epi_apply<bf16>(s, e, m, f, s0, s1);
      }
    }
    cluster_sync();  // peers may still be reading this CTA's partial
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
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k_tc_gemm<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k_tc_gemm<1>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k_tc_gemm<2>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  return e;
}

cudaError_t launch_tc_gemm(const Shape& s, const CUtensorMap* tmW, const CUtensorMap* tmX, int na, const TcPlan& p,
                           const TcGemmArgs& a, bool pdl, cudaStream_t st) {
  const int ntiles = (a.N + 127) / 128;
  dim3 grid(ntiles, p.splits, p.tok_tiles);
  const size_t smem = tc_gemm_smem_bytes(na, p);
  if (na == 2) return launch_ex(k_tc_gemm<2>, grid, dim3(128), smem, st, p.splits, pdl, *tmW, *tmX, s, p, a);
  return launch_ex(k_tc_gemm<1>, grid, dim3(128), smem, st, p.splits, pdl, *tmW, *tmX, s, p, a);
}

}  // namespace pae
