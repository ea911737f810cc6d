// Multi-query decode: T new tokens of every sequence attend in one call, each
// through its own band.  The "Step-3.7-Flash" spec card's architecture notes
// list three extra multi-token-prediction (MTP) layers that speed up decoding;
// the tokens they propose are checked this way.  The band and the cache rule
// are the "Step-3.7-Flash-oQ3e" explainer's
// section 2.2 (a sliding layer keeps the last W tokens; query i sees keys
// i - W < j <= i), the gate its section 2.3.
//
// The cache holds the L0 = L - T earlier tokens (ring slot p mod W, or slot p);
// the new tokens' rotated keys and values come separately, so checking drafts
// never overwrites ring slots an earlier query still needs.  Query t sits at
// position L0 + t.  On a ring, dist(s) = (s - n - 1) mod W numbers the slots
// from the oldest (n = slot of position L0 - 1); query t loses exactly the
// slots with dist <= t, and sees new key j iff t - W < j <= t.
//
// Work split: one CTA per (sequence, kv-head, split of the cache), as in the
// one-query decode, but the M dimension of the m16n8k16 MMAs is now the
// T * G (query, head) rows of the kv-head: warp w owns rows 16w .. 16w + 15
// over every key of the split, so the warps never merge.  One elected thread
// streams 32-key K/V stages with TMA (no producer warp: at 49 KB of stages and
// at most 168 registers, four CTAs share an SM, so the 512 (sequence,
// kv-head) pairs of a 64-sequence batch run in one wave); the last split also
// runs one 16-key block of new tokens, staged into a free stage after the loop.
// Cache bytes are still read once per (sequence, kv-head); the T-fold rows
// raise the tensor work per byte, which stays far below the MMA rate.
#pragma once
#include "decode.cuh"

namespace swa {

namespace decode_mq_detail {

using decode_detail::KB;
using decode_detail::kBoxBytes;
using decode_detail::kStageBytes;
using decode_detail::ldsm_x4;
using decode_detail::ldsm_x4_t;
using decode_detail::mma_bf16;
using decode_detail::sigmoidf_;
using decode_detail::sw128_off;

constexpr int kNewRows = 16;  // new-token block (T <= 16), zero-padded, staged in stage 0
constexpr int kStages = 3;
// resident CTAs per SM: four (49 KB of shared memory each); four m-tiles
// would spill at the register share of four, so they run three per SM
constexpr int ctas_per_sm(int mt) { return mt <= 3 ? 4 : 3; }
static_assert(kNewRows == kDecodeMqMaxT, "one block holds every new token");
static_assert(ctas_per_sm(3) == decode_mq_ctas_per_sm(48) && ctas_per_sm(4) == decode_mq_ctas_per_sm(64),
              "the split plan sees the kernel's occupancy");
static_assert(kStageBytes % 1024 == 0 && kNewRows <= KB, "stage boxes stay 1024-byte aligned and hold the new rows");

struct MqSmem {
  uint8_t stage[kStages][kStageBytes];  // K lo, K hi, V lo, V hi boxes of 32 keys
  uint64_t full[kStages];
  uint64_t empty[kStages];
  int abort_flag;
};

// One warp's 16 rows: Q fragments, output accumulators, running max (log2
// units) and per-lane partial sums of rows g and g + 8.
struct RowState {
  uint32_t qf[8][4];
  float o[16][4];
  float m0, m1, l0, l1;
};

// One block of NK keys: S = Q K^T, masked online softmax, O += P V.  The K/V
// halves lie `box` bytes apart.  vis(kidx, hi) tells whether key kidx of the
// block is visible to row g (hi = 0) or g + 8 (hi = 1).  Keys at or past
// `live`, and key `dead` (a slot outside every query's band, or -1), are
// never visible; their V rows are zeroed in registers, as they may hold NaN
// and 0 * NaN would reach the sum.
template <int NK, bool kMasked, class Vis>
__device__ __forceinline__ void mq_block(RowState& R, uint32_t kbase, uint32_t vbase, uint32_t box, float c,
                                         int lane, int live, int dead, Vis vis) {
  constexpr int NT = NK / 8;
  const int tig = lane & 3;
  // S: the NT accumulation chains advance together, one 32-dim step at a
  // time, so NT independent MMAs are in flight behind each other
  float sc[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
  for (int kk = 0; kk < 8; kk += 2) {
    const int ch = 2 * kk + (lane >> 3);  // 16-byte chunk (8 dims) 0..15
    uint32_t kb[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
      ldsm_x4(kbase + (ch >> 3) * box + sw128_off(nt * 8 + (lane & 7), ch & 7), kb[nt][0], kb[nt][1], kb[nt][2],
              kb[nt][3]);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) mma_bf16(sc[nt], R.qf[kk], kb[nt][0], kb[nt][1]);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) mma_bf16(sc[nt], R.qf[kk + 1], kb[nt][2], kb[nt][3]);
  }
  float p[NT][4];
  float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float v = sc[nt][e] * c;
      p[nt][e] = (!kMasked || vis(nt * 8 + 2 * tig + (e & 1), e >> 1)) ? v : -INFINITY;
    }
    mx0 = fmaxf(mx0, fmaxf(p[nt][0], p[nt][1]));
    mx1 = fmaxf(mx1, fmaxf(p[nt][2], p[nt][3]));
  }
  mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
  mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
  mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
  mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
  const float mn0 = fmaxf(R.m0, mx0), mn1 = fmaxf(R.m1, mx1);
  const float ms0 = mn0 == -INFINITY ? 0.f : mn0, ms1 = mn1 == -INFINITY ? 0.f : mn1;
  const float al0 = fast_exp2(R.m0 - ms0), al1 = fast_exp2(R.m1 - ms1);
  R.m0 = mn0;
  R.m1 = mn1;
  float s0 = 0.f, s1 = 0.f;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    p[nt][0] = fast_exp2(p[nt][0] - ms0);
    p[nt][1] = fast_exp2(p[nt][1] - ms0);
    p[nt][2] = fast_exp2(p[nt][2] - ms1);
    p[nt][3] = fast_exp2(p[nt][3] - ms1);
    s0 += p[nt][0] + p[nt][1];
    s1 += p[nt][2] + p[nt][3];
  }
  R.l0 = R.l0 * al0 + s0;
  R.l1 = R.l1 * al1 + s1;
#pragma unroll
  for (int n = 0; n < 16; ++n) {
    R.o[n][0] *= al0; R.o[n][1] *= al0;
    R.o[n][2] *= al1; R.o[n][3] *= al1;
  }
  const int mi = lane >> 3;
#pragma unroll
  for (int ks = 0; ks < NK / 16; ++ks) {
    uint32_t pa[4];
    pa[0] = pack_bf16x2(p[2 * ks][0], p[2 * ks][1]);
    pa[1] = pack_bf16x2(p[2 * ks][2], p[2 * ks][3]);
    pa[2] = pack_bf16x2(p[2 * ks + 1][0], p[2 * ks + 1][1]);
    pa[3] = pack_bf16x2(p[2 * ks + 1][2], p[2 * ks + 1][3]);
    // this lane's B fragments hold keys k0, k0 + 1 (b0, b2) and k0 + 8, k0 + 9 (b1, b3)
    const int k0 = ks * 16 + 2 * tig;
    auto keep = [&](int k) -> bool { return k < live && k != dead; };
    const uint32_t keep_lo = (keep(k0) ? 0x0000FFFFu : 0u) | (keep(k0 + 1) ? 0xFFFF0000u : 0u);
    const uint32_t keep_hi = (keep(k0 + 8) ? 0x0000FFFFu : 0u) | (keep(k0 + 9) ? 0xFFFF0000u : 0u);
    const bool sanitize = live < NK || (unsigned)dead < (unsigned)NK;
    const int vrow = ks * 16 + (mi & 1) * 8 + (lane & 7);
#pragma unroll
    for (int n = 0; n < 16; n += 2) {
      const int ch = n + (mi >> 1);  // dims 8*ch .. 8*ch+7
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(vbase + (ch >> 3) * box + sw128_off(vrow, ch & 7), b0, b1, b2, b3);
      if (sanitize) {
        b0 &= keep_lo; b2 &= keep_lo;
        b1 &= keep_hi; b3 &= keep_hi;
      }
      mma_bf16(R.o[n], pa, b0, b1);
      mma_bf16(R.o[n + 1], pa, b2, b3);
    }
  }
}

// grid (max_splits, Hkv, B); MT warps of 16 rows each.  Lane 0 of warp 0
// also issues the TMA loads: the first kStages blocks up front, then at the
// top of step t the block t - 1 + kStages into the stage every warp released
// after step t - 1.
template <int MT>
__global__ void __launch_bounds__(MT * 32, ctas_per_sm(MT))
    decode_mq_kernel(const DecodeMqArgs a, const __grid_constant__ CUtensorMap k_map,
                     const __grid_constant__ CUtensorMap v_map) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  MqSmem& sm = *reinterpret_cast<MqSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  allow_dependent_launch();
  grid_dependency_wait();
  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int T = a.T;
  const int L0 = a.seq_lens[b] - T;  // cached tokens before the new ones
  const bool ring = a.window > 0;
  if (L0 < 0 || (!ring && L0 > a.capacity)) {  // uniform over the CTA, before any barrier
    if (threadIdx.x == 0 && split == 0 && kvh == 0) record_error(kErrDecodeMq + (L0 < 0 ? 3 : 4));
    return;
  }
  const int n_cache = ring ? min(L0, a.window) : L0;
  const int n_split = max(1, (n_cache + a.chunk - 1) / a.chunk);
  if (split >= n_split) return;
  const int k_begin = split * a.chunk;
  const int k_end = min(n_cache, k_begin + a.chunk);
  const int n_blocks = k_end > k_begin ? (k_end - k_begin + KB - 1) / KB : 0;
  const bool has_new = split == n_split - 1;
  const int newest = (ring && L0 > 0) ? (L0 - 1) % a.window : 0;  // ring slot of position L0 - 1
  // a full ring's oldest slot (position L0 - W) lies outside every query's band
  const int dead_slot = (ring && L0 >= a.window) ? (newest + 1) % a.window : -1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool issuer = threadIdx.x == 0;
  const int row3 = b * a.Hkv + kvh;
  auto issue = [&](int t) {
    const int s = t % kStages;
    const int key0 = k_begin + t * KB;
    uint8_t* st = sm.stage[s];
    mbar_arrive_expect_tx(&sm.full[s], kStageBytes);
    tma_load_3d(st, &k_map, &sm.full[s], 0, key0, row3);
    tma_load_3d(st + kBoxBytes, &k_map, &sm.full[s], 64, key0, row3);
    tma_load_3d(st + 2 * kBoxBytes, &v_map, &sm.full[s], 0, key0, row3);
    tma_load_3d(st + 3 * kBoxBytes, &v_map, &sm.full[s], 64, key0, row3);
  };
  int issued = 0;
  if (issuer) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], MT);
    }
    sm.abort_flag = 0;
    fence_mbar_init();
    if (n_blocks > 0) {
      prefetch_tensormap(&k_map);
      prefetch_tensormap(&v_map);
    }
    for (; issued < n_blocks && issued < kStages; ++issued) issue(issued);
  }
  __syncthreads();
  volatile int* abort_flag = &sm.abort_flag;

  const int g = lane >> 2, tig = lane & 3;
  const int G = a.G, n_rows = T * G;
  const int r0 = warp * 16 + g, r1 = r0 + 8;
  const bool v0 = r0 < n_rows, v1 = r1 < n_rows;
  const int t0 = v0 ? r0 / G : 0, t1 = v1 ? r1 / G : 0;
  const int h0 = kvh * G + (v0 ? r0 % G : 0), h1 = kvh * G + (v1 ? r1 % G : 0);
  const size_t row0 = ((size_t)b * T + t0) * a.Hq + h0, row1 = ((size_t)b * T + t1) * a.Hq + h1;

  RowState R;
  {
    const uint32_t* q0 = reinterpret_cast<const uint32_t*>(a.q + row0 * kHeadDim);
    const uint32_t* q1 = reinterpret_cast<const uint32_t*>(a.q + row1 * kHeadDim);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const int w0 = kk * 8 + tig;  // 32-bit word of dims (16kk + 2tig, +1)
      R.qf[kk][0] = v0 ? __ldg(q0 + w0) : 0u;
      R.qf[kk][1] = v1 ? __ldg(q1 + w0) : 0u;
      R.qf[kk][2] = v0 ? __ldg(q0 + w0 + 4) : 0u;
      R.qf[kk][3] = v1 ? __ldg(q1 + w0 + 4) : 0u;
    }
  }
#pragma unroll
  for (int n = 0; n < 16; ++n) R.o[n][0] = R.o[n][1] = R.o[n][2] = R.o[n][3] = 0.f;
  R.m0 = R.m1 = -INFINITY;
  R.l0 = R.l1 = 0.f;
  const float c = a.scale_log2;
  const int W = a.window;

  for (int t = 0; t < n_blocks; ++t) {
    const int s = t % kStages;
    if (issuer && t > 0 && issued < n_blocks) {
      // every warp has released step t - 1's stage: refill it
      if (!mbar_wait(&sm.empty[(t - 1) % kStages], ((t - 1) / kStages) & 1, abort_flag)) {
        record_error(kErrDecodeMq + 1);
        *abort_flag = 1;
      } else {
        issue(issued++);
      }
    }
    if (*abort_flag || !mbar_wait(&sm.full[s], (t / kStages) & 1, abort_flag)) {
      record_error(kErrDecodeMq + 2);
      *abort_flag = 1;
      break;
    }
    const uint32_t kbase = smem_u32(sm.stage[s]);
    const uint32_t vbase = kbase + 2 * kBoxBytes;
    const int key0 = k_begin + t * KB;
    const int live = k_end - key0;
    // A block needs masks when it is ragged or, on a ring, holds one of the
    // T oldest slots (dist < T): the first key's dist, or the wrap point
    // (dist 0) inside the block.
    bool masked = live < KB;
    if (ring && !masked) {
      int d_first = key0 - newest - 1;
      if (d_first < 0) d_first += W;
      const int wrap = (newest + 1) % W;
      masked = d_first < T || (wrap > key0 && wrap < key0 + KB);
    }
    if (masked) {
      auto vis = [&](int kidx, int hi) -> bool {
        if (kidx >= live) return false;
        if (!ring) return true;
        int d = key0 + kidx - newest - 1;
        if (d < 0) d += W;
        return d > (hi ? t1 : t0);
      };
      mq_block<KB, true>(R, kbase, vbase, kBoxBytes, c, lane, live, dead_slot < 0 ? -1 : dead_slot - key0, vis);
    } else {
      mq_block<KB, false>(R, kbase, vbase, kBoxBytes, c, lane, KB, -1, [](int, int) -> bool { return true; });
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.empty[s]);
  }
  __syncthreads();  // every warp is past the loop, aborted or not
  if (*abort_flag) {
    // let every copy the issuer started land before the CTA exits
    if (issuer)
      for (int t = issued > kStages ? issued - kStages : 0; t < issued; ++t)
        mbar_wait(&sm.full[t % kStages], (t / kStages) & 1, nullptr, 200000000ull);
    return;
  }

  if (has_new) {
    // every warp is past its last stage read and every load has landed:
    // stage 0 takes the new tokens' K and V rows (zero past T)
    for (int i = threadIdx.x; i < 2 * kNewRows * 16; i += MT * 32) {
      const int tensor = i / (kNewRows * 16), row = (i >> 4) % kNewRows, ch = i & 15;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (row < T) {
        const uint16_t* src = (tensor ? a.v_new : a.k_new) + (((size_t)b * T + row) * a.Hkv + kvh) * kHeadDim;
        v = __ldg(reinterpret_cast<const uint4*>(src) + ch);
      }
      *reinterpret_cast<uint4*>(sm.stage[0] + (tensor * 2 + (ch >> 3)) * kBoxBytes + sw128_off(row, ch & 7)) = v;
    }
    __syncthreads();
    const uint32_t fb = smem_u32(sm.stage[0]);
    auto vis = [&](int j, int hi) -> bool {
      const int tq = hi ? t1 : t0;
      return j <= tq && (!ring || j > tq - W);
    };
    mq_block<kNewRows, true>(R, fb, fb + 2 * kBoxBytes, kBoxBytes, c, lane, kNewRows, -1, vis);
  }

  float l0 = R.l0, l1 = R.l1;
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  if (a.max_splits == 1) {
    if (v0) {
      const float sc = (a.gate ? sigmoidf_(a.gate[row0]) : 1.f) / l0;
      uint32_t* dst = reinterpret_cast<uint32_t*>(a.out + row0 * kHeadDim);
#pragma unroll
      for (int n = 0; n < 16; ++n) dst[n * 4 + tig] = pack_bf16x2(R.o[n][0] * sc, R.o[n][1] * sc);
    }
    if (v1) {
      const float sc = (a.gate ? sigmoidf_(a.gate[row1]) : 1.f) / l1;
      uint32_t* dst = reinterpret_cast<uint32_t*>(a.out + row1 * kHeadDim);
#pragma unroll
      for (int n = 0; n < 16; ++n) dst[n * 4 + tig] = pack_bf16x2(R.o[n][2] * sc, R.o[n][3] * sc);
    }
  } else {
    if (v0) {
      const size_t slot = row0 * a.max_splits + split;
      float2* dst = reinterpret_cast<float2*>(a.part_o + slot * kHeadDim);
#pragma unroll
      for (int n = 0; n < 16; ++n) dst[n * 4 + tig] = make_float2(R.o[n][0], R.o[n][1]);
      if (tig == 0) a.part_ml[slot] = make_float2(R.m0, l0);
    }
    if (v1) {
      const size_t slot = row1 * a.max_splits + split;
      float2* dst = reinterpret_cast<float2*>(a.part_o + slot * kHeadDim);
#pragma unroll
      for (int n = 0; n < 16; ++n) dst[n * 4 + tig] = make_float2(R.o[n][2], R.o[n][3]);
      if (tig == 0) a.part_ml[slot] = make_float2(R.m1, l1);
    }
  }
}

// grid (Hq, T, B), 128 threads: merge the splits of one (sequence, query, q-head).
// A split whose keys all lie outside a query's band left (-inf, 0) and weighs 0.
__global__ void __launch_bounds__(128) decode_mq_combine_kernel(const DecodeMqArgs a) {
  allow_dependent_launch();
  grid_dependency_wait();
  const int h = blockIdx.x, t = blockIdx.y, b = blockIdx.z, d = threadIdx.x;
  const int L0 = a.seq_lens[b] - a.T;
  if (L0 < 0 || (a.window < 0 && L0 > a.capacity)) return;
  const int n_cache = a.window > 0 ? min(L0, a.window) : L0;
  const int n_split = min(a.max_splits, max(1, (n_cache + a.chunk - 1) / a.chunk));
  const size_t row = ((size_t)b * a.T + t) * a.Hq + h;
  const size_t base = row * a.max_splits;
  float M = -INFINITY;
  for (int s = 0; s < n_split; ++s) M = fmaxf(M, a.part_ml[base + s].x);
  float lsum = 0.f, acc = 0.f;
  for (int s = 0; s < n_split; ++s) {
    const float2 ml = a.part_ml[base + s];
    const float f = ml.x == -INFINITY ? 0.f : fast_exp2(ml.x - M);
    lsum += f * ml.y;
    acc += f * a.part_o[(base + s) * kHeadDim + d];
  }
  const float gt = a.gate ? sigmoidf_(a.gate[row]) : 1.f;
  a.out[row * kHeadDim + d] = __bfloat16_as_ushort(__float2bfloat16_rn(acc / lsum * gt));
}

template <int MT>
cudaError_t launch_mq(const DecodeMqArgs& a, const CUtensorMap& k_map, const CUtensorMap& v_map,
                      cudaStream_t stream) {
  const size_t smem = sizeof(MqSmem) + 1024;
  static DeviceOnce setup;
  cudaError_t e = device_once(setup, [&](int, int*) {
    return cudaFuncSetAttribute(decode_mq_kernel<MT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  });
  if (e != cudaSuccess) return e;
  e = launch_kernel(true, decode_mq_kernel<MT>, dim3(a.max_splits, a.Hkv, a.B), dim3(MT * 32), smem, stream, a, k_map,
                       v_map);
  if (e != cudaSuccess || a.max_splits == 1) return e;
  return launch_kernel(true, decode_mq_combine_kernel, dim3(a.Hq, a.T, a.B), dim3(kHeadDim), 0, stream, a);
}

}  // namespace decode_mq_detail

cudaError_t launch_decode_mq(const DecodeMqArgs& a, const CUtensorMap& k_map, const CUtensorMap& v_map,
                             cudaStream_t stream) {
  if (a.B == 0) return cudaSuccess;
  switch ((a.T * a.G + 15) / 16) {
    case 1: return decode_mq_detail::launch_mq<1>(a, k_map, v_map, stream);
    case 2: return decode_mq_detail::launch_mq<2>(a, k_map, v_map, stream);
    case 3: return decode_mq_detail::launch_mq<3>(a, k_map, v_map, stream);
    case 4: return decode_mq_detail::launch_mq<4>(a, k_map, v_map, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace swa
