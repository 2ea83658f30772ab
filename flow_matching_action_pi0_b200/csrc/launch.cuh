// Kernel launch helper: thread-block clusters and programmatic dependent
// launch (PDL) through cudaLaunchKernelEx, plus the device-side PDL and
// cluster primitives the kernels use.
#pragma once

#include <cuda_runtime.h>

namespace pae {

// Launch `kern` with an optional cluster along grid.y and optional PDL (the
// kernel may start while its predecessor in the stream finishes; it must call
// pdl_wait() before reading anything the predecessor writes).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_ex(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                             int cluster_y, bool pdl, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attrs[2];
  unsigned n = 0;
  if (cluster_y > 1) {
    attrs[n].id = cudaLaunchAttributeClusterDimension;
    attrs[n].val.clusterDim.x = 1;
    attrs[n].val.clusterDim.y = (unsigned)cluster_y;
    attrs[n].val.clusterDim.z = 1;
    ++n;
  }
  if (pdl) {
    attrs[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  cfg.attrs = attrs;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Wait until the predecessor grid has completed and its writes are visible
// (returns at once when the kernel was not launched with PDL).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Allow the successor grid to be scheduled (it still waits in pdl_wait()).
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Optional launch trace (built with -DPAE_GRAPH_TRACE; off otherwise): every
// CTA of the projection, attention and token kernels appends one record
// {entered, predecessor wait returned, marks 1-9, left, class | CTA << 8 |
// SM << 40} (%globaltimer, ns; a mark never set stays 0) to a buffer that
// pae_graph_trace_bind_* hands in.  Marks may be set by any thread (shared
// memory, last writer wins); thread 0 writes the record after the kernel's
// final CTA barrier.  Each translation unit holds its own buffer pointer.
#ifdef PAE_GRAPH_TRACE
struct GTraceRec {
  unsigned long long t[15], meta;
};
static __device__ GTraceRec* g_gtrace_buf = nullptr;
static __device__ unsigned int* g_gtrace_ctr = nullptr;
static __device__ unsigned int g_gtrace_cap = 0;
__device__ __forceinline__ unsigned long long gtrace_now() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void gtrace_emit(const unsigned long long* t, int cls) {
  if (threadIdx.x != 0 || g_gtrace_buf == nullptr) return;
  const unsigned i = atomicAdd(g_gtrace_ctr, 1u);
  if (i >= g_gtrace_cap) return;
  unsigned smid;
  asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
  const unsigned long long cta = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
  GTraceRec r;
#pragma unroll
  for (int k = 0; k < 11; ++k) r.t[k] = t[k];
  r.t[11] = gtrace_now();
#pragma unroll
  for (int k = 12; k < 15; ++k) r.t[k] = 0;
  r.meta = (unsigned long long)cls | (cta << 8) | ((unsigned long long)smid << 40);
  g_gtrace_buf[i] = r;
}
static inline cudaError_t gtrace_bind_tu(void* buf, void* ctr, unsigned cap) {
  cudaError_t e = cudaMemcpyToSymbol(g_gtrace_buf, &buf, sizeof(buf));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_gtrace_ctr, &ctr, sizeof(ctr));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_gtrace_cap, &cap, sizeof(cap));
  return e;
}
// GTRACE_BEGIN: marks of thread 0 only (registers); GTRACE_BEGIN_SHARED:
// marks of any thread (88 bytes of static shared memory).
#define GTRACE_BEGIN()                                                   \
  unsigned long long gt_[11] = {gtrace_now(), 0, 0, 0, 0, 0, 0, 0, 0, 0, 0}; \
  (void)gt_
#define GTRACE_BEGIN_SHARED()                                 \
  __shared__ unsigned long long gt_[11];                      \
  if (threadIdx.x == 0) {                                     \
    gt_[0] = gtrace_now();                                    \
    for (int gti_ = 1; gti_ < 11; ++gti_) gt_[gti_] = 0;      \
  }
#define GTRACE_WAITED() \
  do {                  \
    if (threadIdx.x == 0) gt_[1] = gtrace_now(); \
  } while (0)
#define GTRACE_MARK(i) \
  do {                 \
    gt_[1 + (i)] = gtrace_now(); \
  } while (0)
#define GTRACE_END(cls) gtrace_emit(gt_, (cls))
#else
#define GTRACE_BEGIN() \
  do {                 \
  } while (0)
#define GTRACE_BEGIN_SHARED() \
  do {                        \
  } while (0)
#define GTRACE_WAITED() \
  do {                  \
  } while (0)
#define GTRACE_MARK(i) \
  do {                 \
  } while (0)
#define GTRACE_END(cls) \
  do {                  \
  } while (0)
#endif

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_cluster(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ float ld_cluster_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ float4 ld_cluster_f32x4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

__device__ __forceinline__ uint4 ld_cluster_u32x4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared::cluster.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

__device__ __forceinline__ void st_cluster_f32x4(uint32_t addr, float a, float b, float c, float d) {
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}
__device__ __forceinline__ void st_cluster_f32x2(uint32_t addr, float a, float b) {
  asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" ::"r"(addr), "f"(a), "f"(b) : "memory");
}

}  // namespace pae
