// One-query-per-sequence attention over a KV cache, split along the cache
// length ("split-K"), followed by a combine kernel that merges the splits with
// log-sum-exp weights and applies the head gate.
//
// Follows the "Step-3.7-Flash-oQ3e" explainer, section 2.2 (a sliding layer's
// KV cache keeps only the last W tokens; full layers see all history) and
// section 2.3 (per-head sigmoid gate), with the "Step-3.7-Flash" spec card's
// GQA grouping (q-head h reads kv-head h / G).  The ring of a sliding layer
// holds exactly the visible keys, in slot order p mod W; softmax does not
// depend on key order, so slots [0, min(L, W)) are read as they lie.
//
// Work split: one CTA per (sequence b, kv-head, split of `chunk` keys).  The
// CTA serves all G q-heads of its kv-head, so each cache byte is read once.
// A producer warp streams 32-key K and V blocks into shared memory with TMA
// (128-byte swizzle, three-stage mbarrier ring); two consumer warps each take
// 16 keys of every block.  At 48 KB of stages a CTA, four CTAs share an SM,
// so a batch of up to 592 (sequence, kv-head, split) CTAs runs in one wave
// with 192 KB of cache reads in flight per SM.  The G (<= 16) query rows are the M dimension of
// m16n8k16 bf16 MMAs (fp32 accumulate): S = Q K^T, an online softmax over the
// fragment rows with quad shuffles, then O += P V with P re-packed from the S
// fragments.  The bound is HBM bandwidth: 512 cache bytes per key against
// 4 * 16 * 128 tensor FLOPs, so the tensor pipe is never the limit.
#pragma once
#include "swa_internal.cuh"

namespace swa {

namespace decode_detail {

constexpr int KB = kDecodeKeyBlock;        // keys per stage
constexpr int kKeysPerWarp = 16;                    // the k16 of one P.V MMA
constexpr int kConsumerWarps = KB / kKeysPerWarp;   // 2
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kCtasPerSm = 4;
constexpr uint32_t kBoxBytes = KB * 128;   // 32 keys x 64 dims x 2 B
constexpr uint32_t kStageBytes = 4 * kBoxBytes;  // K lo/hi + V lo/hi = 16 KB
constexpr int kMergeStride = kHeadDim + 8;       // floats per merged row (padding vs bank conflicts)
static_assert(KB % kKeysPerWarp == 0 && kBoxBytes % 1024 == 0, "stage boxes must stay 1024-byte aligned");

template <int NS>
struct DecodeSmem {
  uint8_t stage[NS][kStageBytes];
  uint64_t full[NS];
  uint64_t empty[NS];
  float m_part[kConsumerWarps][16];
  float l_part[kConsumerWarps][16];
  int abort_flag;
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Byte offset of (row, 16-byte chunk) inside a [rows][128 B] box written by
// TMA with 128-byte swizzle (box base 1024-byte aligned).
__device__ __forceinline__ uint32_t sw128_off(int row, int chunk) {
  return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ float sigmoidf_(float g) { return 1.f / (1.f + __expf(-g)); }

template <int NS>
__global__ void __launch_bounds__(kThreads, kCtasPerSm) decode_split_kernel(const DecodeArgs a,
                                                                const __grid_constant__ CUtensorMap k_map,
                                                                const __grid_constant__ CUtensorMap v_map) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  DecodeSmem<NS>& sm =
      *reinterpret_cast<DecodeSmem<NS>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  allow_dependent_launch();
  grid_dependency_wait();
  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int L = a.seq_lens[b];
  const int n_vis = (a.window > 0 && L > a.window) ? a.window : L;
  const int k_begin = split * a.chunk;
  // a length beyond the host's max_len breaks the call's contract: the keys
  // past the planned splits are not read, and the error word says so
  if (threadIdx.x == 0 && kvh == 0 && split == a.max_splits - 1 && n_vis > k_begin + a.chunk)
    record_error(kErrDecode + 3);
  if (L < 1 || k_begin >= n_vis) return;  // uniform over the CTA, before any barrier
  const int k_end = min(n_vis, k_begin + a.chunk);
  const int n_blocks = (k_end - k_begin + KB - 1) / KB;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], kConsumerWarps);
    }
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  volatile int* abort_flag = &sm.abort_flag;

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tensormap(&k_map);
      prefetch_tensormap(&v_map);
      const int row3 = b * a.Hkv + kvh;
      int issued = 0;
      for (int t = 0; t < n_blocks; ++t) {
        const int s = t % NS, u = t / NS;
        if (u > 0 && !mbar_wait(&sm.empty[s], (u - 1) & 1, abort_flag)) {
          record_error(kErrDecode + 1);
          *abort_flag = 1;
          break;
        }
        mbar_arrive_expect_tx(&sm.full[s], kStageBytes);
        const int key0 = k_begin + t * KB;
        uint8_t* st = sm.stage[s];
        tma_load_3d(st, &k_map, &sm.full[s], 0, key0, row3);
        tma_load_3d(st + kBoxBytes, &k_map, &sm.full[s], 64, key0, row3);
        tma_load_3d(st + 2 * kBoxBytes, &v_map, &sm.full[s], 0, key0, row3);
        tma_load_3d(st + 3 * kBoxBytes, &v_map, &sm.full[s], 64, key0, row3);
        issued = t + 1;
      }
      if (*abort_flag) {
        // let every copy this warp started land before the CTA exits
        for (int t = issued > NS ? issued - NS : 0; t < issued; ++t)
          mbar_wait(&sm.full[t % NS], (t / NS) & 1, nullptr, 200000000ull);
      }
    }
  } else {
    // ------------------------------------------------------ consumers
    const int g = lane >> 2, tig = lane & 3;
    const int G = a.G;
    // Q fragments (rows = the G q-heads of this kv-head, zero-padded to 16)
    uint32_t qf[8][4];
    {
      const uint32_t* q0 = reinterpret_cast<const uint32_t*>(a.q + ((size_t)b * a.Hq + kvh * G + g) * kHeadDim);
      const uint32_t* q1 = reinterpret_cast<const uint32_t*>(a.q + ((size_t)b * a.Hq + kvh * G + g + 8) * kHeadDim);
      const bool r0 = g < G, r1 = g + 8 < G;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const int w0 = kk * 8 + tig;  // 32-bit word index of dims (16kk + 2tig, +1)
        qf[kk][0] = r0 ? __ldg(q0 + w0) : 0u;
        qf[kk][1] = r1 ? __ldg(q1 + w0) : 0u;
        qf[kk][2] = r0 ? __ldg(q0 + w0 + 4) : 0u;
        qf[kk][3] = r1 ? __ldg(q1 + w0 + 4) : 0u;
      }
    }
    float o[16][4];
#pragma unroll
    for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY;  // running max (log2 units), rows g and g+8
    float l0 = 0.f, l1 = 0.f;              // per-lane partial row sums
    const float c = a.scale_log2;

    for (int t = 0; t < n_blocks; ++t) {
      const int s = t % NS;
      if (!mbar_wait(&sm.full[s], (t / NS) & 1, abort_flag)) {
        record_error(kErrDecode + 2);
        *abort_flag = 1;
        break;
      }
      const uint32_t kbase = smem_u32(sm.stage[s]);
      const uint32_t vbase = kbase + 2 * kBoxBytes;
      const int key_w = k_begin + t * KB + warp * kKeysPerWarp;  // first key of this warp
      const int live = k_end - key_w;                               // keys of this warp still visible
      if (live < kKeysPerWarp) {
        // zero the V rows of keys past the visible range (they may hold NaN)
        uint8_t* vst = sm.stage[s] + 2 * kBoxBytes;
        for (int idx = lane; idx < kKeysPerWarp * 16; idx += 32) {
          const int kr = idx >> 4, ch = idx & 15;
          if (kr >= live) {
            const int row = warp * kKeysPerWarp + kr;
            *reinterpret_cast<uint4*>(vst + (ch >> 3) * kBoxBytes + sw128_off(row, ch & 7)) =
                make_uint4(0, 0, 0, 0);
          }
        }
        __syncwarp();
      }
      // S = Q K^T for this warp's 16 keys: two n-tiles of 8 keys
      float sc[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
        const int krow = warp * kKeysPerWarp + nt * 8 + (lane & 7);
#pragma unroll
        for (int kk = 0; kk < 8; kk += 2) {
          const int ch = 2 * kk + (lane >> 3);  // 16-byte chunk (8 dims) 0..15
          uint32_t b0, b1, b2, b3;
          ldsm_x4(kbase + (ch >> 3) * kBoxBytes + sw128_off(krow, ch & 7), b0, b1, b2, b3);
          mma_bf16(sc[nt], qf[kk], b0, b1);
          mma_bf16(sc[nt], qf[kk + 1], b2, b3);
        }
      }
      // online softmax over the 16 keys (rows g and g+8)
      float x[2][4];
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int kidx = nt * 8 + 2 * tig + (e & 1);
          const float v = kidx < live ? sc[nt][e] * c : -INFINITY;
          x[nt][e] = v;
        }
        mx0 = fmaxf(mx0, fmaxf(x[nt][0], x[nt][1]));
        mx1 = fmaxf(mx1, fmaxf(x[nt][2], x[nt][3]));
      }
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
      const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
      const float ms0 = mn0 == -INFINITY ? 0.f : mn0, ms1 = mn1 == -INFINITY ? 0.f : mn1;
      const float al0 = fast_exp2(m0 - ms0), al1 = fast_exp2(m1 - ms1);
      m0 = mn0;
      m1 = mn1;
      float p[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        p[nt][0] = fast_exp2(x[nt][0] - ms0);
        p[nt][1] = fast_exp2(x[nt][1] - ms0);
        p[nt][2] = fast_exp2(x[nt][2] - ms1);
        p[nt][3] = fast_exp2(x[nt][3] - ms1);
      }
      l0 = l0 * al0 + (p[0][0] + p[0][1] + p[1][0] + p[1][1]);
      l1 = l1 * al1 + (p[0][2] + p[0][3] + p[1][2] + p[1][3]);
#pragma unroll
      for (int n = 0; n < 16; ++n) {
        o[n][0] *= al0; o[n][1] *= al0;
        o[n][2] *= al1; o[n][3] *= al1;
      }
      uint32_t pa[4];
      pa[0] = pack_bf16x2(p[0][0], p[0][1]);
      pa[1] = pack_bf16x2(p[0][2], p[0][3]);
      pa[2] = pack_bf16x2(p[1][0], p[1][1]);
      pa[3] = pack_bf16x2(p[1][2], p[1][3]);
      // O += P V: V rows = this warp's 16 keys, 16 n-tiles of 8 dims
      {
        const int mi = lane >> 3;
        const int vrow = warp * kKeysPerWarp + (mi & 1) * 8 + (lane & 7);
#pragma unroll
        for (int n = 0; n < 16; n += 2) {
          const int ch = n + (mi >> 1);  // dims 8*ch .. 8*ch+7
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(vbase + (ch >> 3) * kBoxBytes + sw128_off(vrow, ch & 7), b0, b1, b2, b3);
          mma_bf16(o[n], pa, b0, b1);
          mma_bf16(o[n + 1], pa, b2, b3);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[s]);
    }

    // ---- merge the four consumer warps through shared memory
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    named_bar_sync(1, kConsumerWarps * 32);  // every warp is done reading the stages
    static_assert(sizeof(float) * kConsumerWarps * 16 * kMergeStride <= sizeof(sm.stage),
                  "the merge reuses the stages");
    if (!*abort_flag) {
      float* mo = reinterpret_cast<float*>(sm.stage[0]);  // [warps][16][kMergeStride], over the idle stages
      float* mine = mo + warp * 16 * kMergeStride;
#pragma unroll
      for (int n = 0; n < 16; ++n) {
        const int d = n * 8 + 2 * tig;
        *reinterpret_cast<float2*>(mine + g * kMergeStride + d) = make_float2(o[n][0], o[n][1]);
        *reinterpret_cast<float2*>(mine + (g + 8) * kMergeStride + d) = make_float2(o[n][2], o[n][3]);
      }
      if (tig == 0) {
        sm.m_part[warp][g] = m0;
        sm.m_part[warp][g + 8] = m1;
        sm.l_part[warp][g] = l0;
        sm.l_part[warp][g + 8] = l1;
      }
    }
    named_bar_sync(1, kConsumerWarps * 32);
    if (!*abort_flag) {
      const float* mo = reinterpret_cast<const float*>(sm.stage[0]);
      // each consumer thread merges two adjacent head dims of every row
      const int d = 2 * threadIdx.x;
      static_assert(2 * 32 * kConsumerWarps == kHeadDim, "two dims per consumer thread");
      for (int r = 0; r < G; ++r) {
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, sm.m_part[w][r]);
        float lsum = 0.f, acc0 = 0.f, acc1 = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
          const float f = sm.m_part[w][r] == -INFINITY ? 0.f : fast_exp2(sm.m_part[w][r] - M);
          lsum += f * sm.l_part[w][r];
          const float2 v = *reinterpret_cast<const float2*>(mo + (w * 16 + r) * kMergeStride + d);
          acc0 += f * v.x;
          acc1 += f * v.y;
        }
        const int h = kvh * G + r;
        if (a.max_splits == 1) {
          const float gt = a.gate ? sigmoidf_(a.gate[(size_t)b * a.Hq + h]) : 1.f;
          const float sc = gt / lsum;
          *reinterpret_cast<uint32_t*>(a.out + ((size_t)b * a.Hq + h) * kHeadDim + d) =
              pack_bf16x2(acc0 * sc, acc1 * sc);
        } else {
          const size_t slot = ((size_t)b * a.Hq + h) * a.max_splits + split;
          *reinterpret_cast<float2*>(a.part_o + slot * kHeadDim + d) = make_float2(acc0, acc1);
          if (d == 0) a.part_ml[slot] = make_float2(M, lsum);
        }
      }
    }
  }
}

// grid (Hq, B), 128 threads: merge the splits of one (sequence, q-head).
__global__ void __launch_bounds__(128) decode_combine_kernel(const DecodeArgs a) {
  allow_dependent_launch();
  grid_dependency_wait();
  const int h = blockIdx.x, b = blockIdx.y, d = threadIdx.x;
  const int L = a.seq_lens[b];
  const int n_vis = (a.window > 0 && L > a.window) ? a.window : L;
  // never past this row's planned partials (a length beyond max_len is
  // recorded by the split kernel)
  const int n_split = min((n_vis + a.chunk - 1) / a.chunk, a.max_splits);
  const size_t base = ((size_t)b * a.Hq + h) * a.max_splits;
  float M = -INFINITY;
  for (int s = 0; s < n_split; ++s) M = fmaxf(M, a.part_ml[base + s].x);
  float lsum = 0.f, acc = 0.f;
  for (int s = 0; s < n_split; ++s) {
    const float2 ml = a.part_ml[base + s];
    const float f = fast_exp2(ml.x - M);
    lsum += f * ml.y;
    acc += f * a.part_o[(base + s) * kHeadDim + d];
  }
  const float gt = a.gate ? sigmoidf_(a.gate[(size_t)b * a.Hq + h]) : 1.f;
  a.out[((size_t)b * a.Hq + h) * kHeadDim + d] = __bfloat16_as_ushort(__float2bfloat16_rn(acc / lsum * gt));
}

constexpr int kStages = 3;

}  // namespace decode_detail

cudaError_t launch_decode(const DecodeArgs& a, const CUtensorMap& k_map, const CUtensorMap& v_map,
                          cudaStream_t stream) {
  if (a.B == 0) return cudaSuccess;
  using namespace decode_detail;
  const size_t smem = sizeof(DecodeSmem<kStages>) + 1024;
  static DeviceOnce setup;
  cudaError_t e = device_once(setup, [&](int, int*) {
    return cudaFuncSetAttribute(decode_split_kernel<kStages>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  });
  if (e != cudaSuccess) return e;
  dim3 grid(a.max_splits, a.Hkv, a.B);
  e = launch_kernel(true, decode_split_kernel<kStages>, grid, dim3(kThreads), smem, stream, a, k_map, v_map);
  if (e != cudaSuccess || a.max_splits == 1) return e;
  return launch_kernel(true, decode_combine_kernel, dim3(a.Hq, a.B), dim3(kHeadDim), 0, stream, a);
}

}  // namespace swa
