// Internal declarations shared by the kernels and the C-ABI layer of
// libswa.so.  Nothing here is part of the public interface (include/swa.h).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "ptx.cuh"

namespace swa {

// Launches a kernel; with `dependent`, with programmatic stream serialization,
// so that it can be scheduled while the previous kernel on the stream
// finishes (its blocks wait in grid_dependency_wait(); see ptx.cuh).  The
// decode-path kernels use it (B200: the batched decode 29.3 -> 27.5 us
// launched one by one); the prefill path does not (it measured slower), and
// its kernels carry no dependency instructions.
template <class... KArgs, class... Args>
cudaError_t launch_kernel(bool dependent, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = dependent ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

// One-time setup per device for a launcher: kernel attributes (the opt-in
// shared memory size) belong to a device context, so a process that drives
// several GPUs sets them on each.  fn(dev, &value) runs once per device
// ordinal, under a lock; value (e.g. the SM count) is returned every call.
constexpr int kMaxSetupDevices = 64;
struct DeviceOnce {
  std::mutex mu;
  uint64_t done = 0;
  int value[kMaxSetupDevices] = {};
};

template <class Fn>
cudaError_t device_once(DeviceOnce& o, Fn fn, int* value_out = nullptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxSetupDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(o.mu);
  if (!((o.done >> dev) & 1ull)) {
    e = fn(dev, &o.value[dev]);
    if (e != cudaSuccess) return e;
    o.done |= 1ull << dev;
  }
  if (value_out) *value_out = o.value[dev];
  return cudaSuccess;
}

constexpr int kHeadDim = 128;
constexpr int kMaxRotaryHalf = kHeadDim / 2;

// Device error codes (kernel * 100 + wait site) recorded by bounded waits.
enum : int {
  kErrPrefill = 100,
  kErrDecode = 200,
  kErrRope = 300,
  kErrDecodeMq = 400,
};

// ------------------------------------------------------------------ RoPE

// Cos/sin table of the prefill: one float2 (cos, sin) per (position i, rotary
// pair k < r/2), stored so that 32 consecutive positions read the same two
// pairs from 512 contiguous bytes: groups of 32 positions, within a group the
// couples of pairs (k/2) in order, within a couple the 32 positions, within a
// position the two pairs.  A warp whose lanes hold 32 consecutive query rows
// then loads a 16-byte (two-pair) slice per lane fully coalesced.
__host__ __device__ __forceinline__ int rope_table_couples(int half) { return (half + 1) >> 1; }
__host__ __device__ __forceinline__ long long rope_table_index(long long i, int k, int half) {
  return ((((i >> 5) * rope_table_couples(half) + (k >> 1)) << 5) + (i & 31)) * 2 + (k & 1);
}
// bytes for positions 0..S-1 (whole groups of 32)
__host__ __device__ __forceinline__ long long rope_table_bytes(long long S, int half) {
  return ((S + 31) >> 5) * rope_table_couples(half) * 32 * 16;
}

struct RopeArgs {
  int B, S, Hq, Hkv;
  int rotary_dim;            // even, 0..128
  int pos0;
  const int32_t* pos;        // [B,S] or nullptr (pos0 + s)
  uint16_t* q;               // [B,S,Hq,D] rotated in place, or nullptr
  const uint16_t* k_src;     // [B,S,Hkv,D] or nullptr
  uint16_t* k_dst;           // rotated keys, [B, dst_rows, Hkv, D] from row dst_row_off (may alias k_src); required with k_src
  int dst_rows;              // rows per sequence of k_dst (0: S)
  int dst_row_off;           // row of k_dst that token 0 of a sequence goes to
  const uint16_t* v;         // [B,S,Hkv,D], for the cache append
  uint16_t* k_cache;         // [B,Hkv,C,D] or nullptr
  uint16_t* v_cache;
  int cache_capacity;        // C
  int window;                // W >= 1 or -1 (slot rule; with pos == nullptr a ring keeps the call's last W positions)
  float2* table;             // cos/sin of positions 0..S-1 (rope_table_index layout), or nullptr
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
  const float2* table;       // cos/sin (rope_table_index layout), when rotary_dim > 0
  const float* gate;         // [B,S,Hq] or nullptr
  int n_q_tiles;             // ceil(S / 128)
  int n_head_pairs;          // ceil(G / 2)
  int q_off;                 // key-space position of query row 0 (keys 0 .. q_off + S - 1); 0 for a whole prefill
  int kv_cache_layout;       // 0: k/v maps {D, Hkv, keys, B}; 1: a KV cache, maps {D, keys, B * Hkv}
};

// q_map / o_map (the bf16 output [B, S, Hq, D]): 4-D {D, Hq, S, B}; k_map /
// v_map: 4-D {D, Hkv, q_off + S, B} (any strides: a KV cache [B, Hkv, C, D]
// is addressed in place); boxes {64, 1, 128, 1}, 128-byte swizzle.  Query row
// r sits at key-space position q_off + r; the cos/sin table, the gate and the
// output rows are indexed by r.
cudaError_t launch_prefill(const PrefillArgs& a, const CUtensorMap& q_map, const CUtensorMap& k_map,
                           const CUtensorMap& v_map, const CUtensorMap& o_map, cudaStream_t stream);

// ------------------------------------------------------ continued prefill

struct KvGatherArgs {
  int B, S, Hkv;
  int h;                     // history tokens gathered per sequence (<= W - 1)
  int pos0;                  // position of the chunk's first token
  int window, capacity;      // the ring: W == C slots
  const uint16_t* k_cache;   // [B, Hkv, C, D]
  const uint16_t* v_cache;
  const uint16_t* v;         // [B, S, Hkv, D] the chunk's values
  uint16_t* k_seq;           // [B, h + S, Hkv, D]: rows 0..h-1 written here
  uint16_t* v_seq;           // [B, h + S, Hkv, D]: all rows written here
};

cudaError_t launch_kv_gather(const KvGatherArgs& a, cudaStream_t stream);

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

constexpr int kDecodeKeyBlock = 32;   // keys per pipeline stage

// --------------------------------------------------- multi-query decode

constexpr int kDecodeMqMaxT = 16;      // new tokens per sequence
constexpr int kDecodeMqMaxRows = 64;   // T * G (query, head) rows per kv-head

struct DecodeMqArgs {
  int B, T, Hq, Hkv, G;
  int window;                // W >= 1 (ring of W slots) or -1 (linear)
  int capacity;              // C
  float scale_log2;
  const uint16_t* q;         // [B,T,Hq,D] rotated
  const float* gate;         // [B,T,Hq] or nullptr
  const uint16_t* k_new;     // [B,T,Hkv,D] rotated keys of the new tokens
  const uint16_t* v_new;     // [B,T,Hkv,D]
  const int32_t* seq_lens;   // [B], counting the T new tokens
  uint16_t* out;             // [B,T,Hq,D]
  int chunk;                 // cache keys per split (multiple of the key block)
  int max_splits;
  float* part_o;             // [B*T*Hq][max_splits][D] (split mode)
  float2* part_ml;           // [B*T*Hq][max_splits]
};

// q_map 4-D {D, Hq, T, B} box {64, G, T, 1} (the (t, g) rows of one kv-head);
// k_map / v_map 3-D {D, C, B*Hkv} box {64, 64, 1}; kn_map / vn_map (the new
// tokens' keys and values) 4-D {D, Hkv, T, B} box {64, 1, 16, 1}; chunk a
// multiple of kDecodeMqKeyBlock.
constexpr int kDecodeMqKeyBlock = 64;
constexpr int kDecodeMqCtasPerSm = 2;
cudaError_t launch_decode_mq(const DecodeMqArgs& a, const CUtensorMap& q_map, const CUtensorMap& k_map,
                             const CUtensorMap& v_map, const CUtensorMap& kn_map, const CUtensorMap& vn_map,
                             cudaStream_t stream);

}  // namespace swa
