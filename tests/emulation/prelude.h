// Test-only host emulation of CUDA thread blocks, included before a kernel source compiled with
// g++: the CUDA keywords become plain C++, the thread and block indices come from the fiber that
// runs, and barriers, warp shuffles and cluster operations call the fiber runtime (fibers.cpp).
#pragma once
#define __global__
#define __launch_bounds__(...)
#define __cluster_dims__(...)
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cmath>
#include <cstring>
#include <cstdint>
#include <functional>
namespace emu {
extern uint3 tid_, bid_;
extern dim3 bdim_, gdim_;
extern int cluster_size;
void syncthreads();
int syncthreads_or(int p);
void syncwarp();
void cluster_sync();
unsigned cluster_rank();
void* cluster_map(void* p, unsigned rank);
uint64_t xchg(uint64_t bits, int src_lane, bool xor_mode);
template <class T> T shfl_xor(unsigned, T v, int lm) {
  uint64_t b = 0; memcpy(&b, &v, sizeof(T)); b = xchg(b, lm, true); T r; memcpy(&r, &b, sizeof(T)); return r;
}
template <class T> T shfl(unsigned, T v, int src) {
  uint64_t b = 0; memcpy(&b, &v, sizeof(T)); b = xchg(b, src, false); T r; memcpy(&r, &b, sizeof(T)); return r;
}
float4* smem();
void* shared_static_bytes(int id, size_t bytes);
template <class T> T& shared_static(int id) { return *static_cast<T*>(shared_static_bytes(id, sizeof(T))); }
unsigned match_any(unsigned long long v);
unsigned ballot(int p);
int lane_id();
template <class T> T shfl_up(unsigned, T v, int d) {
  const int lane = lane_id();
  uint64_t b = 0; memcpy(&b, &v, sizeof(T)); b = xchg(b, lane >= d ? lane - d : lane, false); T r; memcpy(&r, &b, sizeof(T)); return r;
}
void launch(dim3 grid, dim3 block, size_t smem_bytes, std::function<void()> body);
}
namespace cooperative_groups {
struct cluster_group {
  unsigned block_rank() const { return ::emu::cluster_rank(); }
  void sync() const { ::emu::cluster_sync(); }
  template <class T> T* map_shared_rank(T* p, unsigned r) const { return static_cast<T*>(::emu::cluster_map(p, r)); }
};
inline cluster_group this_cluster() { return {}; }
}
#define threadIdx (::emu::tid_)
#define blockIdx (::emu::bid_)
#define blockDim (::emu::bdim_)
#define gridDim (::emu::gdim_)
#define __syncthreads() ::emu::syncthreads()
#define __syncthreads_or(p) ::emu::syncthreads_or(p)
#define __syncwarp(...) ::emu::syncwarp()
#define __shfl_xor_sync(m, v, l) ::emu::shfl_xor(m, v, l)
#define __shfl_sync(m, v, l) ::emu::shfl(m, v, l)
#define __shfl_up_sync(m, v, d) ::emu::shfl_up(m, v, d)
#define __ballot_sync(m, p) ::emu::ballot((p) ? 1 : 0)
#define __ldg(p) (*(p))
#define __ldcs(p) (*(p))
#define __popc(x) __builtin_popcount(x)
#define __ffs(x) __builtin_ffs(x)
#define __match_any_sync(m, v) ::emu::match_any((unsigned long long)(long long)(v))
inline unsigned atomicOr(unsigned* p, unsigned v) { unsigned o = *p; *p |= v; return o; }
inline int atomicAdd(int* p, int v) { int o = *p; *p += v; return o; }
inline float atomicAdd(float* p, float v) { float o = *p; *p += v; return o; }
