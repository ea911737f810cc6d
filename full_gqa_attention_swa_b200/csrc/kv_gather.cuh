// Assembles the key/value sequence a continued prefill chunk of a sliding
// layer attends to: the last h earlier tokens, read from the layer's ring
// cache (position p in slot p mod W; "Step-3.7-Flash-oQ3e" explainer section
// 2.2: the sliding layers keep the last W tokens), followed by the chunk's own
// values.  The chunk's rotated keys are written after the history rows by the
// RoPE pass (rope.cuh, dst_rows / dst_row_off).  Pure data movement: one
// 16-byte lane per (token, kv-head, 16-byte chunk of the 256-byte row).
#pragma once
#include "swa_internal.cuh"

namespace swa {

namespace kv_gather_detail {

constexpr int kLanes = kHeadDim * 2 / 16;  // 16 lanes per 256-byte row

// grid.x covers B * (h + S) * Hkv * 16 lanes
__global__ void __launch_bounds__(256) kv_gather_kernel(const KvGatherArgs a) {
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int lane = (int)(tid % kLanes);
  long long rest = tid / kLanes;
  const int h = (int)(rest % a.Hkv);
  rest /= a.Hkv;
  const int rows = a.h + a.S;
  const int row = (int)(rest % rows);
  const long long b = rest / rows;
  if (b >= a.B) return;
  const size_t dst = ((((size_t)b * rows + row) * a.Hkv + h) * kHeadDim) / 8 + lane;
  if (row < a.h) {
    // history token at position pos0 - h + row, in ring slot position mod W
    const long long p = (long long)a.pos0 - a.h + row;
    const long long slot = p % a.window;
    const size_t src = ((((size_t)b * a.Hkv + h) * a.capacity + slot) * kHeadDim) / 8 + lane;
    reinterpret_cast<uint4*>(a.k_seq)[dst] = reinterpret_cast<const uint4*>(a.k_cache)[src];
    reinterpret_cast<uint4*>(a.v_seq)[dst] = reinterpret_cast<const uint4*>(a.v_cache)[src];
  } else {
    const size_t src = ((((size_t)b * a.S + (row - a.h)) * a.Hkv + h) * kHeadDim) / 8 + lane;
    reinterpret_cast<uint4*>(a.v_seq)[dst] = reinterpret_cast<const uint4*>(a.v)[src];
  }
}

}  // namespace kv_gather_detail

cudaError_t launch_kv_gather(const KvGatherArgs& a, cudaStream_t stream) {
  const long long lanes = (long long)a.B * (a.h + a.S) * a.Hkv * kv_gather_detail::kLanes;
  if (lanes == 0) return cudaSuccess;
  const long long blocks = (lanes + 255) / 256;
  if (blocks > 0x7FFFFFFFll) return cudaErrorInvalidConfiguration;
  return launch_kernel(false, kv_gather_detail::kv_gather_kernel, dim3((unsigned)blocks), dim3(256), 0, stream, a);
}

}  // namespace swa
