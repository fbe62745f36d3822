// trace.cuh -- host-side launch counter and optional per-kernel CUDA-event
// timing (a measurement aid; not thread safe, see include/attn.h).
#pragma once

#include <cuda_runtime.h>

#include <utility>
#include <vector>

enum KernelKind : int {
  KK_DOC_RANGES = 0,
  KK_ROPE_PREP,
  KK_FWD,
  KK_DELTA,
  KK_DKDV,
  KK_DQ,
  KK_DQ_FINALIZE,
  KK_DECODE,
  KK_DECODE_COMBINE,
  KK_GEMM,
  KK_ROPE_GRAD,
  KK_FILL,
  KK_COUNT
};

static const char* const kKernelNames[KK_COUNT] = {
    "doc_ranges", "rope_prep", "fwd", "delta", "dkdv", "dq", "dq_finalize", "decode",
    "decode_combine", "gemm", "rope_grad", "fill"};

namespace trace {

constexpr int kMaxTimed = 16384;

struct Record {
  cudaEvent_t a, b;
  int kind;
};

inline unsigned long long& launches() {
  static unsigned long long n = 0;
  return n;
}
inline bool& enabled() {
  static bool on = false;
  return on;
}
inline std::vector<Record>& pool() {
  static std::vector<Record> p;
  return p;
}
inline int& used() {
  static int u = 0;
  return u;
}

// Call before a kernel launch: counts it and, when timing is on, records the
// opening event on the launch stream. Returns the record index or -1.
inline int begin(int kind, cudaStream_t st) {
  ++launches();
  if (!enabled() || used() >= (int)pool().size()) return -1;
  Record& r = pool()[used()];
  r.kind = kind;
  if (cudaEventRecord(r.a, st) != cudaSuccess) return -1;
  return used()++;
}
inline void end(int idx, cudaStream_t st) {
  if (idx >= 0) cudaEventRecord(pool()[idx].b, st);
}

inline int enable(bool on) {
  if (on && pool().empty()) {
    pool().resize(kMaxTimed);
    for (auto& r : pool()) {
      if (cudaEventCreate(&r.a) != cudaSuccess || cudaEventCreate(&r.b) != cudaSuccess) {
        pool().clear();
        return -1;
      }
    }
  }
  if (on) used() = 0;
  enabled() = on;
  return 0;
}

inline int read(int kind, int* n, double* ms) {
  *n = 0;
  *ms = 0.0;
  for (int i = 0; i < used(); ++i) {
    const Record& r = pool()[i];
    if (r.kind != kind) continue;
    if (cudaEventSynchronize(r.b) != cudaSuccess) return -1;
    float t = 0.f;
    if (cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess) return -1;
    *ms += t;
    ++*n;
  }
  return 0;
}

}  // namespace trace

// Launch with programmatic stream serialization: the kernel may be scheduled
// while its predecessor in the stream is finishing (each kernel waits for its
// predecessor's completion before touching memory, see pdl_wait_and_trigger).
// A launch error is kept for launch_status().
inline cudaError_t& pdl_launch_error() {
  static cudaError_t e = cudaSuccess;
  return e;
}
template <typename... KArgs, typename... Args>
inline void pdl_launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  if (e != cudaSuccess) pdl_launch_error() = e;
}

// pdl_launch for a kernel whose CTAs run as clusters of cluster_x along x.
template <typename... KArgs, typename... Args>
inline void pdl_cluster_launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                               cudaStream_t st, unsigned cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster_x;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  if (e != cudaSuccess) pdl_launch_error() = e;
}

// Wrap one kernel launch: ATTN_LAUNCH(kind, stream, pdl_launch(kernel, grid, block, smem, stream, ...));
#define ATTN_LAUNCH(kind, st, ...)            \
  do {                                        \
    const int _tr = trace::begin((kind), (st)); \
    __VA_ARGS__;                              \
    trace::end(_tr, (st));                    \
  } while (0)
