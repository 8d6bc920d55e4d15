// Device helpers shared by the libmdr kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace mdr {

constexpr int kMaxHalfD = 64;        // D <= 128
constexpr int kMaxSel = 64;          // R + L <= 64

// Device status codes written to the first word of the workspace.
enum DeviceError : int32_t {
  kDevOk = 0,
  kDevWaitTimeout = 1,      // an mbarrier wait ran out of iterations
  kDevBadSelection = 2,     // a selected block id out of range
  kDevMisaligned = 3,       // dynamic shared memory not 1024-byte aligned
};

// Element traits: 16-byte vectors of the storage type.
template <typename T> struct Elem;

template <> struct Elem<float> {
  static constexpr int kVec = 4;
  __device__ static inline void load(const float* p, float* out) {
    float4 v = __ldg(reinterpret_cast<const float4*>(p));
    out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
  }
  __device__ static inline void unpack(const uint4& v, float* out) {
    out[0] = __uint_as_float(v.x); out[1] = __uint_as_float(v.y);
    out[2] = __uint_as_float(v.z); out[3] = __uint_as_float(v.w);
  }
  __device__ static inline void store(float* p, const float* in) {
    *reinterpret_cast<float4*>(p) = make_float4(in[0], in[1], in[2], in[3]);
  }
  __device__ static inline float to_float(float x) { return x; }
};

template <> struct Elem<__nv_bfloat16> {
  static constexpr int kVec = 8;
  __device__ static inline void load(const __nv_bfloat16* p, float* out) {
    uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      out[2 * i] = __uint_as_float(w[i] << 16);
      out[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
  __device__ static inline void unpack(const uint4& v, float* out) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      out[2 * i] = __uint_as_float(w[i] << 16);
      out[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
  __device__ static inline void store(__nv_bfloat16* p, const float* in) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 h = __floats2bfloat162_rn(in[2 * i], in[2 * i + 1]);
      w[i] = *reinterpret_cast<uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  __device__ static inline float to_float(__nv_bfloat16 x) { return __bfloat162float(x); }
};

// Programmatic dependent launch.  Every libmdr kernel is launched with
// launch_pdl, so it may start (set up shared memory, barriers, tensor memory)
// while the previous kernel on the stream drains; before it reads anything an
// earlier kernel wrote it executes grid_dependency_wait(), which returns once
// the previous kernel has completed and its writes are visible.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Lets the next kernel on the stream start before this one completes (its
// grid_dependency_wait() still waits for this kernel's completion and
// writes).  Called after this kernel's own grid_dependency_wait(), so what
// the next kernel reads before its wait was complete before this kernel ran.
__device__ __forceinline__ void grid_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args&&... args) {
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
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

__device__ inline float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Better of two (score, index) pairs: higher score, lower index on equal scores.
__device__ inline bool better(float s0, int i0, float s1, int i1) {
  return s0 > s1 || (s0 == s1 && i0 < i1);
}

// Warp-wide best (score, index); every lane gets the result.
__device__ inline void warp_best(float& s, int& i) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    float so = __shfl_xor_sync(0xffffffffu, s, o);
    int io = __shfl_xor_sync(0xffffffffu, i, o);
    if (better(so, io, s, i)) { s = so; i = io; }
  }
}

}  // namespace mdr
