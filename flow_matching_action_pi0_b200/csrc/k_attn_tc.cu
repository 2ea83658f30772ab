// GQA attention over [cached prefix | action keys] on the tcgen05 tensor cores.
//
// For request b and KV head g, the G query heads x H action tokens that read
// that KV head form G*H query rows (row r = head-in-group * H + token); they
// share every K and V tile, so they are one M dimension of 128-row tiles.
// Keys are the row's slot: prefix positions [0, lens[b]) then this step's H
// action keys at [lens[b], lens[b] + H) (written by the QKV epilogue).  The mask
// reading: every action token sees all valid prefix keys and all H action
// keys; keys past lens[b] + H are masked.
//
// One CTA = (b, g, 128-row query tile, key split).  Per 64-key chunk c:
//   MMA warp   S_c = Q K_c^T  (M=128, N=64, K=head_dim; TMEM, double buffered)
//   8 warps    online softmax on S_c (two threads per row, log2 domain),
//              rescale O in TMEM when the row max grows by more than 2^8
//              (otherwise keep the old reference), write P_c as bf16
//              pairs into a TMEM buffer of its own (32 columns)
//   MMA warp   O += P_c V_c   (M=128, N=head_dim, K=64; A = P_c read from
//              TMEM, V read MN-major from shared memory)
// Warps 0-3 and 8-11 run the softmax and the output (two threads per query
// row: one per 32-key half of the chunk; row = TMEM lane).  Both threads of a
// row read the whole row of S for its maximum (the same value in both, no
// exchange), so the softmax threads share no barrier inside the chunk loop;
// warp 4 streams Q and the K chunks, warp 6 the V chunks (2-slot rings each,
// a K slot refilled as soon as S of its chunk is done); warp 5 issues the MMAs;
// all twelve warps take part in the split-KV merge.
// Key splits (split-KV, for small batches; up to 16, a non-portable cluster
// size) form a thread-block cluster; their
// unnormalised partial O rows, row maxima and sums are merged through
// distributed shared memory in rank order, so the result is bitwise
// reproducible and no partial touches global memory.
#include "internal.h"
#include "launch.cuh"

namespace pae {

namespace {

constexpr int CK = 64;          // keys per chunk
constexpr int QROWS = 128;      // query rows per CTA
constexpr long long kDrainNs = 4000000000LL;

struct AttnSmem {
  uint32_t q_off, k0_off, v0_off, slot, bar_off, ml_off, total;
  // ring slot st of K / V (arithmetic, so no local-memory array is indexed)
  __host__ __device__ uint32_t k_off(int st) const { return k0_off + (uint32_t)st * slot; }
  __host__ __device__ uint32_t v_off(int st) const { return v0_off + (uint32_t)st * slot; }
};

__host__ __device__ inline AttnSmem attn_layout(int d) {
  AttnSmem L;
  const uint32_t qbytes = QROWS * d * 2;   // d/64 boxes of [128][64]
  const uint32_t kvbytes = CK * d * 2;     // d/64 boxes of [64][64]
  L.q_off = 0;
  L.k0_off = qbytes;
  L.v0_off = qbytes + kvbytes;
  L.slot = 2 * kvbytes;                    // [K0 | V0 | K1 | V1]
  L.bar_off = qbytes + 4 * kvbytes;        // (P lives in TMEM, over its S columns)
  L.ml_off = L.bar_off + 256;
  L.total = L.ml_off + QROWS * 12 + 1024;
  return L;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  const uint32_t lo = __bfloat16_as_ushort(f2bf(a));
  const uint32_t hi = __bfloat16_as_ushort(f2bf(b));
  return lo | (hi << 16);
}

// AND-reduction over the threads of named barrier `id` (`n` of them).  Lanes
// may leave a bounded wait at different times: the warp reconverges before the
// warp-aligned barrier instruction.
__device__ __forceinline__ bool named_and(int id, int n, bool v) {
  __syncwarp();
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void named_sync(int id, int n) {
  __syncwarp();
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// TMEM columns: S double-buffered (2 x CK), O (d), P double-buffered (2 x CK/2).
__host__ __device__ inline uint32_t attn_tmem_cols(int d) {
  uint32_t c = 32;
  while ((int)c < 3 * CK + d) c <<= 1;
  return c;
}

__global__ void __launch_bounds__(384, 1)
    k_attn_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, const Shape s, const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int d = s.d;
  const int nbox = d / 64;
  const AttnSmem L = attn_layout(d);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bar_off);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;   // [2]
  uint64_t* v_full = bars + 3;   // [2]
  uint64_t* k_empty = bars + 5;  // [2] K slot free once S of its chunk is done
  uint64_t* s_full = bars + 7;   // [2]
  uint64_t* p_full = bars + 9;    // [2] P buffer j written (chunks j, j + 2, ...)
  uint64_t* o_done = bars + 11;   // [2] PV of the chunks in P buffer j done
  uint64_t* drain = bars + 13;
  uint64_t* v_empty = bars + 14;  // [2] V slot free once PV of its chunk is done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);
  volatile int* s_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);  // [0] abort
  float* s_ml = reinterpret_cast<float*>(smem + L.ml_off);                // [128][2] row max, row sum
  int* s_ok = reinterpret_cast<int*>(smem + L.ml_off + QROWS * 8);        // [128]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x, split = blockIdx.y, bg = blockIdx.z;
  const int b = bg / s.Hkv, g = bg - b * s.Hkv;
  const int GH = s.G * s.H;
  const int n_valid = a.lens[b] + s.H;  // written only by pae_set_prefix, before the loop
  const int kps = a.keys_per_split;
  const int start = split * kps;
  const int end = min(n_valid, start + kps);
  const int nch = end > start ? (end - start + CK - 1) / CK : 0;
  const int slot_row0 = ((a.layer * s.Bmax + b) * s.Hkv + g) * s.Ptot;
  const float scale_log2 = rsqrtf((float)d) * 1.4426950408889634f;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 16; ++i) mbar_init(&bars[i], (i == 9 || i == 10) ? 256 : 1);
    s_flag[0] = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  const uint32_t ncols = attn_tmem_cols(d);
  if (warp == 0) {
    tmem_alloc(tmem_slot, ncols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_launch_dependents();  // after the TMEM is held (see the projection kernel)
  // q and the action keys come from the previous kernel; the prefix keys were
  // written by pae_set_prefix before the loop, so the producers fetch the
  // chunks that lie wholly inside the prefix before waiting (below).
  if (warp != 4 && warp != 6) pdl_wait();
  const int n_prefix = a.lens[b];
  const uint32_t t_s[2] = {tmem, tmem + CK};
  const uint32_t t_o = tmem + 2 * CK;
  const uint32_t t_p[2] = {t_o + (uint32_t)d, t_o + (uint32_t)d + CK / 2};

  // ------------------------------------------------------------ producers
  // Warp 4 streams Q once and the K chunks, warp 6 the V chunks: a K slot is
  // refilled as soon as S of its chunk is done, ahead of the PV that frees V.
  // chunks 0 and 1 (the two ring slots) if they end inside the prefix
  const int npre = nch < 2 ? (start + CK <= n_prefix ? nch : 0)
                            : (start + 2 * CK <= n_prefix ? 2 : (start + CK <= n_prefix ? 1 : 0));
  if (warp == 4) {
    if (lane == 0)
      for (int c = 0; c < npre; ++c) {
        mbar_arrive_expect_tx(&k_full[c], CK * d * 2);
        for (int x = 0; x < nbox; ++x)
          tma_load_2d(smem + L.k_off(c) + x * CK * 128, &tmK, x * 64, slot_row0 + start + c * CK, &k_full[c]);
      }
    __syncwarp();
    pdl_wait();
  }
  if (warp == 6) {
    if (lane == 0)
      for (int c = 0; c < npre; ++c) {
        mbar_arrive_expect_tx(&v_full[c], CK * d * 2);
        for (int x = 0; x < nbox; ++x)
          tma_load_2d(smem + L.v_off(c) + x * CK * 128, &tmV, x * 64, slot_row0 + start + c * CK, &v_full[c]);
      }
    __syncwarp();
    pdl_wait();
  }
  if (warp == 4 && lane == 0 && nch > 0) {
    const uint32_t kvbytes = CK * d * 2;
    mbar_arrive_expect_tx(q_full, QROWS * d * 2);
    const int qrow0 = bg * GH + qt * QROWS;
    for (int x = 0; x < nbox; ++x) tma_load_2d(smem + L.q_off + x * QROWS * 128, &tmQ, x * 64, qrow0, q_full);
    int issued = npre;
    for (int c = npre; c < nch; ++c) {
      const int st = c & 1;
      if (c >= 2 && !mbar_wait(&k_empty[st], ((c >> 1) & 1) ^ 1, a.err.wait_ns)) {
        s_flag[0] = 1;
        set_error(a.err, DEV_TIMEOUT);
        break;
      }
      const int krow = slot_row0 + start + c * CK;
      mbar_arrive_expect_tx(&k_full[st], kvbytes);
      for (int x = 0; x < nbox; ++x) tma_load_2d(smem + L.k_off(st) + x * CK * 128, &tmK, x * 64, krow, &k_full[st]);
      issued = c + 1;
    }
    if (!mbar_wait(q_full, 0, kDrainNs)) set_error(a.err, DEV_DRAIN);
    for (int c = issued > 2 ? issued - 2 : 0; c < issued; ++c)
      if (!mbar_wait(&k_full[c & 1], (c >> 1) & 1, kDrainNs)) set_error(a.err, DEV_DRAIN);
  }
  if (warp == 6 && lane == 0 && nch > 0) {
    const uint32_t kvbytes = CK * d * 2;
    int issued = npre;
    for (int c = npre; c < nch; ++c) {
      const int st = c & 1;
      if (c >= 2 && !mbar_wait(&v_empty[st], ((c >> 1) & 1) ^ 1, a.err.wait_ns)) {
        s_flag[0] = 1;
        set_error(a.err, DEV_TIMEOUT);
        break;
      }
      const int krow = slot_row0 + start + c * CK;
      mbar_arrive_expect_tx(&v_full[st], kvbytes);
      for (int x = 0; x < nbox; ++x) tma_load_2d(smem + L.v_off(st) + x * CK * 128, &tmV, x * 64, krow, &v_full[st]);
      issued = c + 1;
    }
    for (int c = issued > 2 ? issued - 2 : 0; c < issued; ++c)
      if (!mbar_wait(&v_full[c & 1], (c >> 1) & 1, kDrainNs)) set_error(a.err, DEV_DRAIN);
  }

  // ------------------------------------------------------------ MMA (warp 5)
  if (warp == 5 && lane == 0 && nch > 0) {
    const uint32_t idesc_s = idesc_bf16(QROWS, CK);
    const uint32_t idesc_o = idesc_bf16(QROWS, d, 0, 1);
    const uint32_t q_base = smem_u32(smem + L.q_off);
    bool good = mbar_wait(q_full, 0, a.err.wait_ns);
    // descriptors are built once per operand and stepped in 16-byte units
    const uint64_t q_desc = sw128_desc(q_base, 16, 1024);
    auto issue_s = [&](int c) -> bool {
      const int st = c & 1;
      if (!mbar_wait(&k_full[st], (c >> 1) & 1, a.err.wait_ns)) return false;
      tc_fence_after();
      const uint64_t k_desc = sw128_desc(smem_u32(smem + L.k_off(st)), 16, 1024);
#pragma unroll 4
      for (int k16 = 0; k16 < d / 16; ++k16) {
        const uint32_t x = (uint32_t)k16 >> 2, w = ((uint32_t)k16 & 3u) * 32u;
        umma_bf16(t_s[st], desc_add(q_desc, x * QROWS * 128u + w), desc_add(k_desc, x * CK * 128u + w), idesc_s,
                  k16 > 0 ? 1u : 0u);
      }
      umma_commit(&s_full[st]);
      umma_commit(&k_empty[st]);
      return true;
    };
    if (good) good = issue_s(0);
    if (good && nch > 1) good = issue_s(1);
    for (int c = 0; good && c < nch; ++c) {
      const int st = c & 1;
      if (!mbar_wait(&p_full[st], (c >> 1) & 1, a.err.wait_ns) ||
          !mbar_wait(&v_full[st], (c >> 1) & 1, a.err.wait_ns)) {
        good = false;
        break;
      }
      tc_fence_after();
      const uint64_t v_desc = sw128_desc(smem_u32(smem + L.v_off(st)), CK * 128, 1024);
      // A = P in TMEM: 16 keys per MMA = 8 columns of bf16 pairs
#pragma unroll
      for (int k16 = 0; k16 < CK / 16; ++k16)
        umma_bf16_tmem_a(t_o, t_p[st] + k16 * 8u, desc_add(v_desc, k16 * 16u * 128u), idesc_o,
                         (c > 0 || k16 > 0) ? 1u : 0u);
      umma_commit(&o_done[st]);
      umma_commit(&v_empty[st]);
      if (c + 2 < nch) good = issue_s(c + 2);
    }
    if (!good) {
      s_flag[0] = 1;
      set_error(a.err, DEV_TIMEOUT);
    }
    // every MMA this thread issued must finish before TMEM is freed
    umma_commit(drain);
    if (!mbar_wait(drain, 0, kDrainNs)) set_error(a.err, DEV_DRAIN);
  }
  __syncwarp();

  // ------------------------------------------------------------ softmax
  // Warps 0-3 and 8-11: thread = (query row r = TMEM lane, column half h);
  // half h owns key columns [32h, 32h + 32) of each chunk and output columns
  // [h d/2, (h+1) d/2).  The two halves of a row agree on the running
  // reference maximum through shared memory (s_ml as [2][128] exchange
  // slots, two barriers per chunk); each keeps its own partial row sum, added
  // in a fixed order at the end.  Decisions that guard a named barrier are
  // taken CTA-uniformly over the 256 softmax threads (bar.red.and).
  const bool smx = warp < 4 || warp >= 8;
  if (smx) {
  const int h = warp >= 8 ? 1 : 0;
  const int r = (warp & 3) * 32 + lane;  // query row within the tile (TMEM lane)
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
  const int oc0 = h * (d / 2), oc1 = oc0 + d / 2;  // this half's output columns
  float m_run = -INFINITY, l_run = 0.f;
  bool ok = true;
  for (int c = 0; c < nch; ++c) {
    const int st = c & 1;
    // warp-uniform: the warp's collectives below need every lane
    const bool w1 = __all_sync(0xffffffffu, mbar_wait(&s_full[st], (c >> 1) & 1, a.err.wait_ns));
    if (!w1 || s_flag[0] != 0) {
      ok = false;
      s_flag[0] = 1;  // every thread stops at its next check
      break;
    }
    tc_fence_after();
    // this half's 32 scores, and the other half's for the row maximum (the
    // maximum is exact in any order, so both threads of the row agree)
    float sv[CK / 2], so[CK / 2];
    tmem_ld16(t_s[st] + lane_off + h * 32, sv);
    tmem_ld16(t_s[st] + lane_off + h * 32 + 16, sv + 16);
    tmem_ld16(t_s[st] + lane_off + (1 - h) * 32, so);
    tmem_ld16(t_s[st] + lane_off + (1 - h) * 32 + 16, so + 16);
    tmem_ld_wait();
    const int vc = min(CK, end - (start + c * CK));
    // row maximum as a tree (a chain of 64 dependent max operations would be
    // the longest latency of the chunk at two warps per scheduler)
#pragma unroll
    for (int j = 0; j < CK / 2; ++j) {
      sv[j] = j + h * 32 < vc ? sv[j] * scale_log2 : -INFINITY;
      so[j] = j + (1 - h) * 32 < vc ? so[j] * scale_log2 : -INFINITY;
    }
    float mt[CK / 2];
#pragma unroll
    for (int j = 0; j < CK / 2; ++j) mt[j] = fmaxf(sv[j], so[j]);
#pragma unroll
    for (int w = CK / 4; w >= 1; w >>= 1)
#pragma unroll
      for (int j = 0; j < w; ++j) mt[j] = fmaxf(mt[j], mt[j + w]);
    const float cmax = mt[0];
    // Lazy rescaling: the reference maximum moves only when the row maximum
    // grows by more than 8 (a factor 256), so O is rescaled in TMEM rarely.
    // Probabilities then lie in [0, 256]; the final O / l is the same.
    const float mx = cmax > m_run + 8.f ? cmax : m_run;
    const float alpha = exp2f(m_run - mx);  // 1 when unchanged; 0 on the first chunk
#pragma unroll
    for (int j = 0; j < CK / 2; ++j) sv[j] = exp2f(sv[j] - mx);
    // row sum as a fixed tree (bitwise reproducible)
#pragma unroll
    for (int j = 0; j < CK / 2; ++j) mt[j] = sv[j];
#pragma unroll
    for (int w = CK / 4; w >= 1; w >>= 1)
#pragma unroll
      for (int j = 0; j < w; ++j) mt[j] += mt[j + w];
    const float psum = mt[0];
    l_run = l_run * alpha + psum;
    m_run = mx;
    // P goes into its own buffer; PV of chunk c - 2, which read the previous
    // P there, finished before S of chunk c did (commits complete in issue
    // order).
    bool good = true;
    if (good && c > 0 && __any_sync(0xffffffffu, alpha < 1.f)) {
      // O may be rescaled only once PV of the previous chunk has landed in it.
      good = __all_sync(0xffffffffu, mbar_wait(&o_done[st ^ 1], ((c - 1) >> 1) & 1, a.err.wait_ns));
      if (good) {
        tc_fence_after();
        for (int jj = oc0; jj < oc1; jj += 16) {
          float ov[16];
          tmem_ld16(t_o + lane_off + jj, ov);
          tmem_ld_wait();
#pragma unroll
          for (int t = 0; t < 16; ++t) ov[t] *= alpha;
          tmem_st16(t_o + lane_off + jj, ov);
        }
        tmem_st_wait();
      }
    }
    if (!good) s_flag[0] = 1;  // every thread stops at the next uniform check
    // P row in TMEM: keys 32h .. 32h + 31 as bf16 pairs in columns 16h .. 16h + 15
    {
      float pk[16];
#pragma unroll
      for (int q = 0; q < 16; ++q) pk[q] = __uint_as_float(pack_bf16x2(sv[2 * q], sv[2 * q + 1]));
      tmem_st16(t_p[st] + lane_off + h * 16, pk);
      tmem_st_wait();
    }
    if (vc < CK) {
      // Masked keys have P = 0, but 0 * (NaN or Inf) in V would still poison O:
      // zero the V rows past the valid keys once their load has landed.
      const bool w3 = mbar_wait(&v_full[st], (c >> 1) & 1, kDrainNs);
      if (w3) {
        uint8_t* vbase = smem + L.v_off(st);
        const int rows = CK - vc;
        for (int i = h * QROWS + r; i < rows * nbox * 8; i += 2 * QROWS) {
          const int rr = vc + i / (nbox * 8), rem = i % (nbox * 8), x = rem / 8, ch = rem % 8;
          *reinterpret_cast<uint4*>(vbase + x * CK * 128 + rr * 128 + ch * 16) = make_uint4(0, 0, 0, 0);
        }
      } else {
        s_flag[0] = 1;
      }
      fence_proxy_async_smem();  // the zeroed V rows are read by the tensor cores
    }
    tc_fence_before();
    mbar_arrive(&p_full[st]);
  }
  if (!ok || s_flag[0]) set_error(a.err, DEV_TIMEOUT);
  // PVs complete in issue order: the last chunk's commit covers them all
  if (nch > 0 && ok) ok = mbar_wait(&o_done[(nch - 1) & 1], ((nch - 1) >> 1) & 1, kDrainNs);
  ok = named_and(1, 256, ok) && s_flag[0] == 0;  // CTA-uniform among the 256 softmax threads
  tc_fence_after();
  // row sum = half 0 + half 1 (the exchange slots are free: both passed the barrier)
  s_ml[h * QROWS + r] = l_run;
  named_sync(1, 256);
  const float l_tot = s_ml[r] + s_ml[QROWS + r];
  named_sync(1, 256);

  // ------------------------------------------------------------ output (single split)
  const int nsplit = gridDim.y;
  if (nsplit == 1) {
    const int rq = qt * QROWS + r;
    const bool row_valid = rq < GH;
    const int hl = rq / s.H, ti = rq - hl * s.H;
    bf16* orow = reinterpret_cast<bf16*>(a.o) + (size_t)(b * s.H + ti) * s.attn_dim + (g * s.G + hl) * d;
    const float inv = l_tot > 0.f ? 1.f / l_tot : 0.f;
    if (ok) {
      for (int jj = oc0; jj < oc1; jj += 16) {
        float ov[16];
        tmem_ld16(t_o + lane_off + jj, ov);
        tmem_ld_wait();
        if (row_valid && nch > 0) {
          uint32_t pk[8];
#pragma unroll
          for (int t = 0; t < 8; ++t) pk[t] = pack_bf16x2(ov[2 * t] * inv, ov[2 * t + 1] * inv);
          uint4* dst = reinterpret_cast<uint4*>(orow + jj);
          dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
      }
    }
  } else if (h == 0) {
    s_ok[r] = ok ? 1 : 0;
    s_ml[2 * r] = m_run;
    s_ml[2 * r + 1] = l_tot;
  }
  }  // softmax warps

  if (gridDim.y > 1) {
    // Split-KV merge inside the cluster of key splits.  Every CTA parks its
    // unnormalised O rows as bf16 (row stride d + 8, bank-conflict free; the
    // Q and K/V buffers are idle now) and its row max / sum in shared memory;
    // CTA rank r then merges rows [r*R, r*R+R) over all ranks in rank order.
    // Distributed shared memory moves a few tens of GB/s per SM, so the rows
    // travel in bf16 (the weights and the sum stay fp32) and each (row, rank)
    // weight exp2(m_q - M) / L is formed once, not per column.
    __syncthreads();  // all MMAs and TMEM reads of this CTA are done
    const int ldb = d + 8;
    bf16* red = reinterpret_cast<bf16*>(smem);
    float* tbl = reinterpret_cast<float*>(smem + (size_t)QROWS * ldb * 2);  // [R][S] (m, l), then weights
    if (smx) {
      const int h = warp >= 8 ? 1 : 0;
      const int r = (warp & 3) * 32 + lane;
      const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
      const bool has = s_ok[r] && nch > 0;
      for (int j = h * (d / 2); j < (h + 1) * (d / 2); j += 16) {
        float ov[16];
        if (__all_sync(0xffffffffu, s_ok[(warp & 3) * 32] != 0) && nch > 0) {
          tmem_ld16(t_o + lane_off + j, ov);
          tmem_ld_wait();
        }
        uint32_t pk[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) pk[t] = has ? pack_bf16x2(ov[2 * t], ov[2 * t + 1]) : 0u;
        uint4* dst = reinterpret_cast<uint4*>(red + r * ldb + j);
        dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
      }
      if (!has && h == 0) {
        s_ml[2 * r] = -INFINITY;
        s_ml[2 * r + 1] = 0.f;
      }
    }
    cluster_sync();
    const int S = gridDim.y;
    const uint32_t rank = cluster_rank();
    const int R = QROWS / S;
    const uint32_t red_base = smem_u32(red), ml_base = smem_u32(s_ml);
    // (max, sum) of every (row, rank) once, then the row's weights
    if ((int)threadIdx.x < R * S) {
      const int rr = threadIdx.x / S, q = threadIdx.x - rr * S;
      const uint32_t ra = map_cluster(ml_base + (uint32_t)(((int)rank * R + rr) * 8), (uint32_t)q);
      tbl[2 * threadIdx.x] = ld_cluster_f32(ra);
      tbl[2 * threadIdx.x + 1] = ld_cluster_f32(ra + 4);
    }
    __syncthreads();
    float* wt = tbl + 2 * R * S;  // [R][S]
    if ((int)threadIdx.x < R) {
      const float* e = tbl + 2 * threadIdx.x * S;
      float M = -INFINITY;
      for (int q = 0; q < S; ++q) M = fmaxf(M, e[2 * q]);
      float wsum = 0.f;
      for (int q = 0; q < S; ++q)
        if (e[2 * q + 1] > 0.f) wsum = fmaf(exp2f(e[2 * q] - M), e[2 * q + 1], wsum);
      const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
      for (int q = 0; q < S; ++q)
        wt[threadIdx.x * S + q] = e[2 * q + 1] > 0.f ? exp2f(e[2 * q] - M) * inv : 0.f;
    }
    __syncthreads();
    const int per_row = d / 8;  // 16-byte column groups
    for (int el = threadIdx.x; el < R * per_row; el += blockDim.x) {
      const int rr = el / per_row, c8 = el - rr * per_row;
      const int row = (int)rank * R + rr;
      const int rq = qt * QROWS + row;
      if (rq >= GH) continue;
      // every rank's loads first (they pipeline), then the merge in rank order
      uint4 vs[16];
#pragma unroll
      for (int q = 0; q < 16; ++q)
        if (q < S) vs[q] = ld_cluster_u32x4(map_cluster(red_base + (uint32_t)((row * ldb + c8 * 8) * 2), (uint32_t)q));
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        if (q >= S) continue;
        const float w = wt[rr * S + q];
        const uint32_t u[4] = {vs[q].x, vs[q].y, vs[q].z, vs[q].w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          acc[2 * t] = fmaf(w, __uint_as_float(u[t] << 16), acc[2 * t]);
          acc[2 * t + 1] = fmaf(w, __uint_as_float(u[t] & 0xFFFF0000u), acc[2 * t + 1]);
        }
      }
      const int hl = rq / s.H, ti = rq - hl * s.H;
      bf16* orow = reinterpret_cast<bf16*>(a.o) + (size_t)(b * s.H + ti) * s.attn_dim + (g * s.G + hl) * d;
      *reinterpret_cast<uint4*>(orow + c8 * 8) = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                                                            pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
    }
    cluster_sync();  // peers may still be reading this CTA's partial
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, ncols);
}

}  // namespace

size_t attn_tc_smem_bytes(int d) { return attn_layout(d).total; }

cudaError_t attn_tc_init() {
  cudaError_t e = cudaFuncSetAttribute(k_attn_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k_attn_tc, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  return e;
}

cudaError_t launch_attn_tc(const Shape& s, const CUtensorMap* tmQ, const CUtensorMap* tmK, const CUtensorMap* tmV,
                           const AttnPlan& p, const AttnArgs& a, int B, bool pdl, cudaStream_t st) {
  dim3 grid(p.qtiles, p.splits, B * s.Hkv);
  return launch_ex(k_attn_tc, grid, dim3(384), attn_tc_smem_bytes(s.d), st, p.splits, pdl, *tmQ, *tmK, *tmV, s,
                   a);
}

}  // namespace pae
