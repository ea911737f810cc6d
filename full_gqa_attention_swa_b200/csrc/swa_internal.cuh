// Internal declarations shared by the kernels and the C-ABI layer of
// libswa.so.  Nothing here is part of the public interface (include/swa.h).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ptx.cuh"

namespace swa {

constexpr int kHeadDim = 128;
constexpr int kMaxRotaryHalf = kHeadDim / 2;

// Device error codes (kernel * 100 + wait site) recorded by bounded waits.
enum : int {
  kErrPrefill = 100,
  kErrDecode = 200,
  kErrRope = 300,
};

// ------------------------------------------------------------------ RoPE

struct RopeArgs {
  int B, S, Hq, Hkv;
  int rotary_dim;            // even, 0..128
  int pos0;
  const int32_t* pos;        // [B,S] or nullptr (pos0 + s)
  uint16_t* q;               // [B,S,Hq,D] rotated in place, or nullptr
  const uint16_t* k_src;     // [B,S,Hkv,D] or nullptr
  uint16_t* k_dst;           // [B,S,Hkv,D] rotated keys (may alias k_src); required with k_src
  const uint16_t* v;         // [B,S,Hkv,D], for the cache append
  uint16_t* k_cache;         // [B,Hkv,C,D] or nullptr
  uint16_t* v_cache;
  int cache_capacity;        // C
  int window;                // W >= 1 or -1 (slot rule)
  float2* table;             // [S][rotary_dim/2] (cos, sin) of positions 0..S-1, or nullptr
  int rotate;                // 0: theta == 0 or rotary_dim == 0 (copies only)
  double inv_freq[kMaxRotaryHalf];
};

cudaError_t launch_rope(const RopeArgs& a, cudaStream_t stream);

// --------------------------------------------------------------- prefill

struct PrefillArgs {
  int B, S, Hq, Hkv, G;      // G = Hq / Hkv
  int window;                // W >= 1 or -1
  int rotary_dim;            // rotary dims applied to Q in-kernel (0: none)
  float scale_log2;          // softmax_scale * log2(e)
  const float2* table;       // [S][rotary_dim/2] cos/sin, when rotary_dim > 0
  const float* gate;         // [B,S,Hq] or nullptr
  int n_q_tiles;             // ceil(S / 128)
  int n_head_pairs;          // ceil(G / 2)
};

// q_map / o_map: 4-D {D, Hq, S, B}; k_map / v_map: 4-D {D, Hkv, S, B};
// boxes {64, 1, 128, 1}, 128-byte swizzle.
cudaError_t launch_prefill(const PrefillArgs& a, const CUtensorMap& q_map, const CUtensorMap& k_map,
                           const CUtensorMap& v_map, const CUtensorMap& o_map, cudaStream_t stream);

// ---------------------------------------------------------------- decode

struct DecodeArgs {
  int B, Hq, Hkv, G;
  int window;                // W >= 1 or -1
  int capacity;              // C
  float scale_log2;
  const uint16_t* q;         // [B,Hq,D] rotated
  const float* gate;         // [B,Hq] or nullptr
  const int32_t* seq_lens;   // [B]
  uint16_t* out;             // [B,Hq,D]
  int chunk;                 // keys per split (multiple of the key block)
  int max_splits;            // splits per sequence the workspace holds
  float* part_o;             // [B][Hq][max_splits][D] (split mode)
  float2* part_ml;           // [B][Hq][max_splits]   (m in log2 units, l)
};

// kv maps: 3-D {D, C, B*Hkv}, boxes {64, KB, 1}, 128-byte swizzle.
cudaError_t launch_decode(const DecodeArgs& a, const CUtensorMap& k_map, const CUtensorMap& v_map,
                          cudaStream_t stream);

constexpr int kDecodeKeyBlock = 64;   // keys per pipeline stage

}  // namespace swa
