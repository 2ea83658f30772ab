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
// One CTA = (b, g, 128-row query tile, key split).  Per chunk c of CK keys
// (CK = 64 or 128, a template parameter):
//   MMA warp   S_c = Q K_c^T  (M=128, N=CK, K=head_dim; TMEM, double
//              buffered: chunk c in S buffer c % 2)
//   16 warps   online softmax on S_c (four threads per row, log2 domain),
//              rescale O in TMEM when the row max grows by more than 2^8
//              (otherwise keep the old reference), write P_c as bf16 pairs
//              over the first CK/2 columns of S_c's own buffer
//   MMA warp   O += P_c V_c   (M=128, N=head_dim, K=CK; A = P_c read from
//              TMEM, V read MN-major from shared memory)
// Warps 0-3 and 8-19 run the softmax and the output (four threads per query
// row, one per CK/4-key quarter of the chunk; row = TMEM lane); four warps
// per scheduler hide more of the softmax's latency chain (TMEM load, maximum
// exchange, exp2, TMEM store) than two.  The four parts of a row meet once
// per chunk at a shared-memory exchange of their maxima.  Warp 4 streams Q
// and the K chunks, warp 6 the V chunks, through rings of 128/CK slots of CK
// keys (the same shared memory either way): K of chunk c is loaded once S of
// the chunk that last used its slot is done, V once that chunk's PV is done.
// Long key ranges take CK = 128 (half the chunks, each S with N = 128);
// a split of only 128 keys takes two 64-key chunks, whose softmax and PV
// overlap.  Warp 5 issues the MMAs; all twenty warps take part in the
// split-KV merge.
// Key splits (split-KV, for small batches; up to 8) form a thread-block
// cluster: each writes its unnormalised partial O rows, row maxima and sums
// to a scratch slot in global memory (L2), and after one cluster barrier the
// ranks merge disjoint row ranges in rank order, so the result is bitwise
// reproducible.
#include "internal.h"
#include "launch.cuh"

namespace pae {

namespace {

constexpr int QROWS = 128;      // query rows per CTA
constexpr int RING_KEYS = 128;  // keys of K (and of V) held in shared memory
constexpr long long kDrainNs = 4000000000LL;
constexpr int kMaxSplits = kAttnMaxSplits;  // key splits per cluster

struct AttnSmem {
  uint32_t q_off, k_off, v_off, bar_off, ml_off, total;
};

// K ring, V ring: RING_KEYS keys each, as 128/CK slots of d/64 boxes [CK][64]
// (slot j at j * CK * d * 2 bytes from the ring's start).
__host__ __device__ inline AttnSmem attn_layout(int d) {
  AttnSmem L;
  const uint32_t qbytes = QROWS * d * 2;       // d/64 boxes of [128][64]
  const uint32_t ringbytes = RING_KEYS * d * 2;
  L.q_off = 0;
  L.k_off = qbytes;
  L.v_off = qbytes + ringbytes;
  L.bar_off = qbytes + 2 * ringbytes;          // (P lives in TMEM, over its S columns)
  L.ml_off = L.bar_off + 256;
  L.total = L.ml_off + QROWS * 48 + 1024;
  return L;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  const uint32_t lo = __bfloat16_as_ushort(f2bf(a));
  const uint32_t hi = __bfloat16_as_ushort(f2bf(b));
  return lo | (hi << 16);
}

// 2^x by the hardware approximation (relative error about 2^-22; results
// below 2^-126 flush to zero, far under the bf16 rounding of P).
__device__ __forceinline__ float ex2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
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

// TMEM columns: S double-buffered (2 x CK, P written over the first half of
// its chunk's buffer), O (d).
template <int CK>
__host__ __device__ inline uint32_t attn_tmem_cols(int d) {
  uint32_t c = 32;
  while ((int)c < 2 * CK + d) c <<= 1;
  return c;
}

// 32 lanes x 32 bit, 8 / 16 consecutive columns per thread.
__device__ __forceinline__ void tmem_st8u(uint32_t taddr, const uint32_t* v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(v[0]),
               "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}
__device__ __forceinline__ void tmem_st16u(uint32_t taddr, const uint32_t* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

template <int CK>
__global__ void __launch_bounds__(640, 1)
    k_attn_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, const Shape s, const AttnArgs a) {
  constexpr int NSLOT = RING_KEYS / CK;  // ring slots: chunk c in slot c % NSLOT
  constexpr int HALVES = CK / 64;        // 64-key boxes per chunk
  constexpr int KP = CK / 4;             // keys per softmax part
  GTRACE_BEGIN_SHARED();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int d = s.d;
  const int nbox = d / 64;
  const AttnSmem L = attn_layout(d);
  // Barrier phases count uses: the K / V slot barriers complete once per use
  // of their slot (chunk c: slot c % NSLOT, parity (c / NSLOT) & 1), the
  // per-buffer ones (S, P, PV) once per use of their buffer (chunk c: buffer
  // c & 1, parity (c >> 1) & 1).
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bar_off);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;    // [NSLOT] K chunk landed
  uint64_t* v_full = bars + 3;    // [NSLOT] V chunk landed
  uint64_t* k_empty = bars + 5;   // [NSLOT] K slot free once S of its chunk is done
  uint64_t* s_full = bars + 7;    // [2] S buffer j computed
  uint64_t* p_full = bars + 9;    // [2] P written over S buffer j (chunks j, j + 2, ...)
  uint64_t* o_done = bars + 11;   // [2] PV of the chunk in buffer j done
  uint64_t* drain = bars + 13;
  uint64_t* v_empty = bars + 14;  // [NSLOT] V slot free once PV of its chunk is done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);
  volatile int* s_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);  // [0] abort
  float* s_l = reinterpret_cast<float*>(smem + L.ml_off);   // [4][128] partial row sums
  float* s_pm = s_l + 4 * QROWS;                            // [2][4][128] partial maxima

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
    for (int i = 0; i < 16; ++i) mbar_init(&bars[i], (i == 9 || i == 10) ? 512 : 1);
    s_flag[0] = 0;
    s_flag[1] = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  const uint32_t ncols = attn_tmem_cols<CK>(d);
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
  GTRACE_WAITED();
  const int n_prefix = a.lens[b];
  const uint32_t t_s0 = tmem;                  // S (then P) of chunk parity st at t_s0 + st * CK
  const uint32_t t_o = tmem + 2 * CK;

  // ------------------------------------------------------------ producers
  // Warp 4 streams Q once and the K chunks, warp 6 the V chunks.  A chunk
  // arrives as CK/64 boxes of 64 keys (64-row boxes; a second one lands 8 KB
  // into each 16 KB box region, a whole number of 1024-byte swizzle atoms).
  // The first RING_KEYS keys' boxes that lie wholly inside the prefix (written
  // before the loop) are fetched before waiting for the previous kernel, the
  // rest after it; a chunk's barrier expects all of its bytes once.
  const uint32_t kvbytes = CK * d * 2;  // one chunk of K (or V)
  auto load_piece = [&](uint32_t ring, const CUtensorMap* tm, uint64_t* bar, int c, int h) {
    const uint32_t off = ring + (uint32_t)(c % NSLOT) * kvbytes + (uint32_t)h * 64u * 128u;
    for (int x = 0; x < nbox; ++x)
      tma_load_2d(smem + off + x * CK * 128, tm, x * 64, slot_row0 + start + c * CK + h * 64, bar + (c % NSLOT));
  };
  // 64-key pieces fetched early (pieces 0, 1 = keys [start, start + 128)),
  // only those of chunks that exist
  const int npre_p = min(min(nch * HALVES, 2), start + 128 <= n_prefix ? 2 : start + 64 <= n_prefix ? 1 : 0);
  if (warp == 4 || warp == 6) {
    if (lane == 0) {
      const bool is_k = warp == 4;
      for (int i = 0; i < npre_p; ++i) {
        const int c = i / HALVES, h = i % HALVES;
        if (h == 0) mbar_arrive_expect_tx((is_k ? k_full : v_full) + c, kvbytes);
        load_piece(is_k ? L.k_off : L.v_off, is_k ? &tmK : &tmV, is_k ? k_full : v_full, c, h);
      }
    }
    __syncwarp();
    pdl_wait();
  }
  if ((warp == 4 || warp == 6) && lane == 0 && nch > 0) {
    const bool is_k = warp == 4;
    uint64_t* full = is_k ? k_full : v_full;
    uint64_t* empty = is_k ? k_empty : v_empty;  // S (K) or PV (V) of the slot's previous chunk done
    const CUtensorMap* tm = is_k ? &tmK : &tmV;
    const uint32_t ring = is_k ? L.k_off : L.v_off;
    if (is_k) {
      mbar_arrive_expect_tx(q_full, QROWS * d * 2);
      const int qrow0 = bg * GH + qt * QROWS;
      for (int x = 0; x < nbox; ++x) tma_load_2d(smem + L.q_off + x * QROWS * 128, &tmQ, x * 64, qrow0, q_full);
    }
    int issued = 0;
    for (int c = 0; c < nch; ++c) {
      const int slot = c % NSLOT, use = c / NSLOT;
      if (use > 0 && !mbar_wait(empty + slot, (use & 1) ^ 1, a.err.wait_ns)) {
        s_flag[0] = 1;
        set_error(a.err, DEV_TIMEOUT);
        break;
      }
      const int p0 = c * HALVES;  // this chunk's first piece
      if (p0 >= npre_p) mbar_arrive_expect_tx(full + slot, kvbytes);
      for (int h = 0; h < HALVES; ++h)
        if (p0 + h >= npre_p) load_piece(ring, tm, full, c, h);
      issued = c + 1;
    }
    // Loads still in flight must land before this CTA may exit: only the last
    // NSLOT chunks' can be (every earlier one was consumed by an MMA that
    // completed).
    if (is_k && !mbar_wait(q_full, 0, kDrainNs)) set_error(a.err, DEV_DRAIN);
    for (int c = issued > NSLOT ? issued - NSLOT : 0; c < issued; ++c)
      if (!mbar_wait(full + c % NSLOT, (c / NSLOT) & 1, kDrainNs)) set_error(a.err, DEV_DRAIN);
  }

  // ------------------------------------------------------------ MMA (warp 5)
  if (warp == 5 && lane == 0 && nch > 0) {
    const uint32_t idesc_s = idesc_bf16(QROWS, CK);
    const uint32_t idesc_o = idesc_bf16(QROWS, d, 0, 1);
    const uint32_t q_base = smem_u32(smem + L.q_off);
    bool good = mbar_wait(q_full, 0, a.err.wait_ns);
    // descriptors are built once per operand and stepped in 16-byte units
    const uint64_t q_desc = sw128_desc(q_base, 16, 1024);
    const uint64_t k_desc = sw128_desc(smem_u32(smem + L.k_off), 16, 1024);
    const uint64_t v_desc = sw128_desc(smem_u32(smem + L.v_off), CK * 128, 1024);
    const uint32_t slot_bytes = (uint32_t)CK * (uint32_t)d * 2u;
    // S of chunk c into buffer c & 1.  That buffer last held P of chunk c - 2:
    // its PV must be complete first (waited on explicitly, not left to the
    // issue order).
    auto issue_s = [&](int c) -> bool {
      const int st = c & 1, slot = c % NSLOT;
      if (!mbar_wait(k_full + slot, (c / NSLOT) & 1, a.err.wait_ns)) return false;
      if (c >= 2 && !mbar_wait(&o_done[st], ((c >> 1) & 1) ^ 1, a.err.wait_ns)) return false;
      tc_fence_after();
#pragma unroll 4
      for (int k16 = 0; k16 < d / 16; ++k16) {
        const uint32_t x = (uint32_t)k16 >> 2, w = ((uint32_t)k16 & 3u) * 32u;
        umma_bf16(t_s0 + (uint32_t)(st * CK), desc_add(q_desc, x * QROWS * 128u + w),
                  desc_add(k_desc, slot * slot_bytes + x * CK * 128u + w), idesc_s, k16 > 0 ? 1u : 0u);
      }
      umma_commit(&s_full[st]);
      umma_commit(k_empty + slot);
      return true;
    };
    // Order: S of the next chunk first (the softmax needs it as soon as the
    // current chunk's is done), then PV of the current chunk once its P is in.
    if (good) good = issue_s(0);
    for (int c = 0; good && c < nch; ++c) {
      const int st = c & 1, slot = c % NSLOT;
      if (c + 1 < nch && !(good = issue_s(c + 1))) break;
      if (!mbar_wait(&p_full[st], (c >> 1) & 1, a.err.wait_ns) ||
          !mbar_wait(v_full + slot, (c / NSLOT) & 1, a.err.wait_ns)) {
        good = false;
        break;
      }
      tc_fence_after();
      // A = P in TMEM (over S buffer st): 16 keys per MMA = 8 columns of bf16 pairs
#pragma unroll
      for (int k16 = 0; k16 < CK / 16; ++k16)
        umma_bf16_tmem_a(t_o, t_s0 + (uint32_t)(st * CK) + k16 * 8u,
                         desc_add(v_desc, slot * slot_bytes + k16 * 16u * 128u), idesc_o, (c > 0 || k16 > 0) ? 1u : 0u);
      umma_commit(&o_done[st]);
      umma_commit(v_empty + slot);
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
  // Sixteen warps (0-3 and 8-19): thread = (query row r = TMEM lane, part p
  // of 4); part p owns key columns [KP p, KP p + KP) of each chunk, the P
  // columns [KP p / 2, KP (p + 1) / 2) (its keys as bf16 pairs: the A operand
  // of the chunk's PV MMAs for those keys) and output columns
  // [p d/4, (p+1) d/4).  P
  // overwrites S columns that other parts of the row read: every part has its
  // S in registers before the barrier below, and P is written after it.  The
  // four parts of a row agree on the chunk maximum through shared memory
  // (s_pm[chunk parity][part][row]; the maximum is exact in any order), with
  // one barrier over the 512 softmax threads per chunk that also takes the
  // CTA-uniform go / stop decision (bar.red.and); each part keeps its own
  // partial row sum, added in part order at the end.
  const bool smx = warp < 4 || warp >= 8;
  if (smx) {
  const int part = warp < 4 ? 0 : (warp - 4) >> 2;
  const int r = (warp & 3) * 32 + lane;  // query row within the tile (TMEM lane)
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
  const int oc0 = part * (d / 4), oc1 = oc0 + d / 4;  // this part's output columns
  float m_run = -INFINITY, l_run = 0.f;
  bool ok = true;
  for (int c = 0; c < nch; ++c) {
    const int st = c & 1;
    const bool got = mbar_wait(&s_full[st], (c >> 1) & 1, a.err.wait_ns);
    __syncwarp();
    tc_fence_after();
    float sv[KP];
#pragma unroll
    for (int j = 0; j < KP; j += 16) tmem_ld16(t_s0 + (uint32_t)(st * CK) + lane_off + part * KP + j, sv + j);
    tmem_ld_wait();
#pragma unroll
    for (int j = 0; j < KP; j += 16) reg_fence16(sv + j);
    const int vc = min(CK, end - (start + c * CK));
    // Masking (the last chunk only) and the maximum work on the raw scores:
    // the scale is positive, so max(scale x) = scale max(x), and the scale
    // then rides in the FMA that feeds exp2.
    if (vc < CK) {
#pragma unroll
      for (int j = 0; j < KP; ++j) sv[j] = j + part * KP < vc ? sv[j] : -INFINITY;
    }
    float mt[KP / 2];
#pragma unroll
    for (int j = 0; j < KP / 2; ++j) mt[j] = fmaxf(sv[j], sv[j + KP / 2]);
#pragma unroll
    for (int w = KP / 4; w >= 1; w >>= 1)
#pragma unroll
      for (int j = 0; j < w; ++j) mt[j] = fmaxf(mt[j], mt[j + w]);
    s_pm[(st * 4 + part) * QROWS + r] = mt[0];
    // every part's maximum is in place, and all 512 threads go on or all stop
    if (!named_and(1, 512, got && s_flag[0] == 0)) {
      ok = false;
      break;
    }
    const float* pm = s_pm + st * 4 * QROWS + r;
    const float cmax = fmaxf(fmaxf(pm[0], pm[QROWS]), fmaxf(pm[2 * QROWS], pm[3 * QROWS])) * scale_log2;
    // Lazy rescaling: the reference maximum moves only when the row maximum
    // grows by more than 8 (a factor 256), so O is rescaled in TMEM rarely.
    // Probabilities then lie in [0, 256]; the final O / l is the same.
    const float mx = cmax > m_run + 8.f ? cmax : m_run;
    const float alpha = ex2_ftz(m_run - mx);  // 1 when unchanged; 0 on the first chunk
    const float nmx = -mx;
#pragma unroll
    for (int j = 0; j < KP; ++j) sv[j] = ex2_ftz(fmaf(sv[j], scale_log2, nmx));
    // row sum as a fixed tree (bitwise reproducible)
#pragma unroll
    for (int j = 0; j < KP / 2; ++j) mt[j] = sv[j] + sv[j + KP / 2];
#pragma unroll
    for (int w = KP / 4; w >= 1; w >>= 1)
#pragma unroll
      for (int j = 0; j < w; ++j) mt[j] += mt[j + w];
    l_run = l_run * alpha + mt[0];
    m_run = mx;
    // P goes over S of this chunk; PV of chunk c - 2, which read the previous
    // P there, completed before S of chunk c was issued.
    if (c > 0 && __any_sync(0xffffffffu, alpha < 1.f)) {
      // O may be rescaled only once PV of the previous chunk has landed in it.
      const bool good = __all_sync(0xffffffffu, mbar_wait(&o_done[st ^ 1], ((c - 1) >> 1) & 1, a.err.wait_ns));
      if (good) {
        tc_fence_after();
        for (int jj = oc0; jj < oc1; jj += 16) {
          float ov[16];
          tmem_ld16(t_o + lane_off + jj, ov);
          tmem_ld_wait();
          reg_fence16(ov);
#pragma unroll
          for (int t = 0; t < 16; ++t) ov[t] *= alpha;
          tmem_st16(t_o + lane_off + jj, ov);
        }
        tmem_st_wait();
      } else {
        s_flag[0] = 1;  // every softmax thread stops at the next chunk's barrier
      }
    }
    {
      uint32_t pk[KP / 2];
#pragma unroll
      for (int q = 0; q < KP / 2; ++q) pk[q] = pack_bf16x2(sv[2 * q], sv[2 * q + 1]);
      if constexpr (KP == 32)
        tmem_st16u(t_s0 + (uint32_t)(st * CK) + lane_off + part * 16, pk);
      else
        tmem_st8u(t_s0 + (uint32_t)(st * CK) + lane_off + part * 8, pk);
      tmem_st_wait();
    }
    if (vc < CK) {
      // Masked keys have P = 0, but 0 * (NaN or Inf) in V would still poison O:
      // zero the V rows past the valid keys once their load has landed.
      const bool w3 = mbar_wait(v_full + c % NSLOT, (c / NSLOT) & 1, kDrainNs);
      if (w3) {
        uint8_t* vbase = smem + L.v_off + (c % NSLOT) * kvbytes;
        const int rows = CK - vc;
        for (int i = part * QROWS + r; i < rows * nbox * 8; i += 4 * QROWS) {
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
  if (!ok) set_error(a.err, DEV_TIMEOUT);
  // PVs complete in issue order: the last chunk's commit covers them all
  if (nch > 0 && ok) ok = mbar_wait(&o_done[(nch - 1) & 1], ((nch - 1) >> 1) & 1, kDrainNs);
  ok = named_and(1, 512, ok && s_flag[0] == 0);  // CTA-uniform among the 512 softmax threads
  if (threadIdx.x == 0) s_flag[1] = ok ? 1 : 0;  // for the split-KV merge (read after a CTA barrier)
  tc_fence_after();
  // row sum = the four parts' sums in part order
  s_l[part * QROWS + r] = l_run;
  named_sync(1, 512);
  const float l_tot = ((s_l[r] + s_l[QROWS + r]) + s_l[2 * QROWS + r]) + s_l[3 * QROWS + r];

  // ------------------------------------------------------------ output (single split)
  const int nsplit = gridDim.y;
  if (nsplit == 1) {
    const int rq = qt * QROWS + r;
    const bool row_valid = rq < GH;
    const int hl = rq / s.H, ti = rq - hl * s.H;
    bf16* orow = reinterpret_cast<bf16*>(a.o) + (size_t)(b * s.H + ti) * s.attn_dim + (g * s.G + hl) * d;
    const float inv = l_tot > 0.f ? 1.f / l_tot : 0.f;
    if (ok) {
      // 32 columns per TMEM round trip (16 when a part has only 16: d = 64)
      for (int jj = oc0; jj < oc1; jj += 32) {
        const bool two = jj + 16 < oc1;  // uniform
        float ov[32];
        tmem_ld16(t_o + lane_off + jj, ov);
        if (two) tmem_ld16(t_o + lane_off + jj + 16, ov + 16);
        tmem_ld_wait();
        reg_fence16(ov);
        reg_fence16(ov + 16);
        if (row_valid && nch > 0) {
          uint32_t pk[16];
#pragma unroll
          for (int t = 0; t < 16; ++t) pk[t] = pack_bf16x2(ov[2 * t] * inv, ov[2 * t + 1] * inv);
          uint4* dst = reinterpret_cast<uint4*>(orow + jj);
          dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          if (two) {
            dst[2] = make_uint4(pk[8], pk[9], pk[10], pk[11]);
            dst[3] = make_uint4(pk[12], pk[13], pk[14], pk[15]);
          }
        }
      }
    }
  } else {
    // Split-KV: the row (max, sum) goes to this CTA's scratch slot now; the
    // unnormalised O rows are parked in shared memory below and written out
    // row-contiguously.  Rows without keys (or after a stop) have (-inf, 0).
    const int slot = (blockIdx.z * gridDim.x + qt) * nsplit + split;
    if (part == 0)
      a.part_ml[(size_t)slot * QROWS + r] = (ok && nch > 0) ? make_float2(m_run, l_tot) : make_float2(-INFINITY, 0.f);
  }
  }  // softmax warps

  if (gridDim.y > 1) {
    // Split-KV merge inside the cluster of key splits, through L2.  Every CTA
    // parks its unnormalised O rows as bf16 in shared memory (row stride
    // d + 8, bank-conflict free; Q and the K/V ring are idle now: every MMA
    // and every load has completed) and copies them to its scratch slot with
    // row-contiguous 16-byte stores (coalesced; zeros for a CTA without keys,
    // so the merge reads only defined values).  After one cluster barrier
    // (its release / acquire at cluster scope orders these writes before the
    // peers' reads), CTA rank r merges rows [r*R, r*R+R) over all ranks in
    // rank order, so the result is bitwise reproducible.  An SM moves about
    // 60 GB/s into L2 and 90-170 GB/s out of it, against a few tens of GB/s
    // over distributed shared memory.
    const int S = gridDim.y;
    const int slot = (blockIdx.z * gridDim.x + qt) * S + split;
    const int ldb = d + 8;
    bf16* red = reinterpret_cast<bf16*>(smem);
    __syncthreads();  // every MMA and TMEM read of this CTA is done; s_ok is final
    const bool has = s_flag[1] != 0 && nch > 0;  // CTA-uniform
    if (smx) {
      const int part = warp < 4 ? 0 : (warp - 4) >> 2;
      const int r = (warp & 3) * 32 + lane;
      const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
      for (int j = part * (d / 4); j < (part + 1) * (d / 4); j += 16) {
        float ov[16];
        if (has) {
          tmem_ld16(t_o + lane_off + j, ov);
          tmem_ld_wait();
          reg_fence16(ov);
        }
        uint32_t pk[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) pk[t] = has ? pack_bf16x2(ov[2 * t], ov[2 * t + 1]) : 0u;
        uint4* dst = reinterpret_cast<uint4*>(red + r * ldb + j);
        dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
      }
    }
    __syncthreads();
    {
      const int per_row = d / 8;  // 16-byte column groups
      bf16* prow = a.part_o + (size_t)slot * QROWS * d;
      for (int el = threadIdx.x; el < QROWS * per_row; el += blockDim.x) {
        const int row = el / per_row, c8 = el - row * per_row;
        *reinterpret_cast<uint4*>(prow + (size_t)row * d + c8 * 8) =
            *reinterpret_cast<const uint4*>(red + row * ldb + c8 * 8);
      }
    }
    cluster_sync();
    GTRACE_MARK(1);  // every rank's partial is in L2
    const int R = QROWS / S;
    const int row0 = (int)cluster_rank() * R;
    const int slot0 = slot - split;
    const int per_row = d / 8;
    for (int el = threadIdx.x; el < R * per_row; el += blockDim.x) {
      const int rr = el / per_row, c8 = el - rr * per_row;
      const int row = row0 + rr;
      const int rq = qt * QROWS + row;
      if (rq >= GH) continue;
      // every rank's rows and statistics are requested first (one L2 round
      // trip), then the weights exp2(m_q - M) / L and the merge in rank order
      uint4 vs[kMaxSplits];
      float2 ml[kMaxSplits];
#pragma unroll
      for (int q = 0; q < kMaxSplits; ++q)
        if (q < S) {
          vs[q] = __ldcg(reinterpret_cast<const uint4*>(a.part_o + ((size_t)(slot0 + q) * QROWS + row) * d + c8 * 8));
          ml[q] = __ldcg(a.part_ml + (size_t)(slot0 + q) * QROWS + row);
        }
      float M = -INFINITY;
#pragma unroll
      for (int q = 0; q < kMaxSplits; ++q)
        if (q < S) M = fmaxf(M, ml[q].x);
      float wsum = 0.f;
#pragma unroll
      for (int q = 0; q < kMaxSplits; ++q)
        if (q < S && ml[q].y > 0.f) wsum = fmaf(exp2f(ml[q].x - M), ml[q].y, wsum);
      const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int q = 0; q < kMaxSplits; ++q) {
        if (q >= S || !(ml[q].y > 0.f)) continue;
        const float w = exp2f(ml[q].x - M) * inv;
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
    GTRACE_MARK(2);  // merged rows written
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, ncols);
  GTRACE_END(4);
}

}  // namespace

size_t attn_tc_smem_bytes(int d) { return attn_layout(d).total; }

template <int CK>
cudaError_t attn_init_one() {
  // 1 KB under the 227 KB limit leaves room for a little static shared memory
  cudaError_t e = cudaFuncSetAttribute(k_attn_tc<CK>, cudaFuncAttributeMaxDynamicSharedMemorySize, 226 * 1024);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k_attn_tc<CK>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  return e;
}

cudaError_t attn_tc_init() {
  cudaError_t e = attn_init_one<64>();
  if (e == cudaSuccess) e = attn_init_one<128>();
  return e;
}

cudaError_t launch_attn_tc(const Shape& s, const CUtensorMap* tmQ, const CUtensorMap* tmK, const CUtensorMap* tmV,
                           const AttnPlan& p, const AttnArgs& a, int B, bool pdl, cudaStream_t st) {
  dim3 grid(p.qtiles, p.splits, B * s.Hkv);
  if (p.chunk != 64 && p.chunk != 128) return cudaErrorInvalidValue;
  if (a.keys_per_split % p.chunk != 0) return cudaErrorInvalidValue;
  if (p.chunk == 128)
    return launch_ex(k_attn_tc<128>, grid, dim3(640), attn_tc_smem_bytes(s.d), st, p.splits, pdl, *tmQ, *tmK, *tmV,
                     s, a);
  return launch_ex(k_attn_tc<64>, grid, dim3(640), attn_tc_smem_bytes(s.d), st, p.splits, pdl, *tmQ, *tmK, *tmV, s,
                   a);
}

}  // namespace pae

#ifdef PAE_GRAPH_TRACE
// Trace builds only: hand this file's kernels the launch-trace buffer.
extern "C" int pae_graph_trace_bind_attn(void* buf, void* ctr, unsigned cap) {
  return (int)pae::gtrace_bind_tu(buf, ctr, cap);
}
#endif
