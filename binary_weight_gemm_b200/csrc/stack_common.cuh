// stack_common.cuh -- the layer list and the grid-wide barrier of the persistent
// layer-stack kernels (linear_stack.cu: bf16 warp-level MMA blocks, any M <= 16;
// linear_stack_i8.cu: int8 warp-level MMA on staged activation limbs, M <= 2).
//
// Each layer is  Y = [(X ⊙ b^T) W_sign^T] ⊙ a^T  ("1bit量化", blog.zerodtree.com,
// "proposition 1").  A layer flagged `barrier` reads an output of an earlier layer
// of the list; it starts a barrier group, and the layers between two barriers run
// back to back.
#pragma once

#include <cstdint>

#include "ob_device.cuh"
#include "ob_internal.h"

namespace ob {

struct StackLayer {
  const uint16_t* X;
  const uint32_t* S;
  const float* iscale;
  const float* oscale;
  void* Y;
  int64_t K, N;
  int32_t y_dtype;
  int32_t barrier;  // wait for every earlier layer of the list before this one
  int32_t nb;       // 32-row blocks: ceil(N / 32)
  int32_t vec;      // the sign rows allow 16-byte copies
  // Tagged outputs (int8 form, dataflow launches only): each output also written as a
  // 32-bit word kTagMark | bf16 bits into tag_out, which a consuming layer of the same
  // launch polls (tag_in) instead of waiting at a grid barrier.  Null otherwise.
  uint32_t* tag_out;
  const uint32_t* tag_in;
};

constexpr int kStackMaxLayers = 320;  // 320 x 88 B of kernel parameters

struct StackParams {
  int n;
  int64_t M;
  unsigned* bar;  // [0] arrivals, [1] abort
  unsigned* err;
  int dataflow;   // tagged outputs replace the grid barriers (see StackLayer::tag_out)
  StackLayer L[kStackMaxLayers];
};

// The one- and two-token int8 tensor-core stack (linear_stack_i8.cu): M <= 2 and one
// 16-row tile of every layer fits its 80 KB weight buffer (K <= 40960).
bool stack_i8_supported(const StackParams& p);
cudaError_t launch_stack_i8(const StackParams& p, const LaunchCtx& c);

#ifdef __CUDACC__
__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// All CTAs arrive; returns false (on every thread of the CTA) if the wait ran out
// or another CTA aborted.  The wait is bounded: a CTA that gives up records a
// timeout in the error word and sets the abort word, which makes every other CTA
// leave at its next barrier.
struct NoSideWork {
  __device__ void operator()() const {}
};

// `side` runs on every thread but thread 0 while thread 0 waits (work that needs no
// results of this barrier, e.g. prefetches for later groups).
template <class Side = NoSideWork>
__device__ __forceinline__ bool grid_barrier(unsigned* bar, unsigned target, unsigned* err, int* s_ok,
                                             const Side& side = Side()) {
  __syncthreads();
  if (threadIdx.x != 0) side();
  if (threadIdx.x == 0) {
    __threadfence();  // this CTA's outputs before its arrival
    atomicAdd(bar, 1u);
    int ok = 1;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
      if (ld_acquire_gpu(bar) >= target) break;
      if ((it & 31u) == 0u) {
        if (ld_acquire_gpu(bar + 1) != 0u) {
          ok = 0;
          break;
        }
        if (globaltimer_ns() - t0 > OB_WAIT_LIMIT_NS || it > (1u << 30)) {
          record_error(err, OB_DEVERR_TIMEOUT);
          atomicExch(bar + 1, 1u);
          ok = 0;
          break;
        }
      }
    }
    __threadfence();
    *s_ok = ok;
  }
  __syncthreads();
  return *s_ok != 0;
}

// The first layer index after the barrier group that starts at l.
__device__ __forceinline__ int group_end(const StackParams& p, int l) {
  int e = l + 1;
  while (e < p.n && !p.L[e].barrier) ++e;
  return e;
}
#endif

}  // namespace ob
