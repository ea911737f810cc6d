// Prefill attention on sm_100a: RoPE'd Q, banded causal mask, GQA, online
// softmax, P.V and the per-head sigmoid gate, with tcgen05 tensor-core MMAs
// accumulating in tensor memory and TMA loads into shared memory.
//
// Follows the "Step-3.7-Flash-oQ3e" explainer: section 2.2 (sliding-window
// causal mask of W keys on sliding layers, plain causal mask on full layers)
// and section 2.3 (per-layer rope theta, partial rotary, head-wise sigmoid
// gate); the "Step-3.7-Flash" spec card's GQA groups; the "Muse-Glimmer-30B-
// 6bit" explainer's theta = 0 (no rotation) on full layers.
//
// One CTA = 128 query rows x two q-heads of the same kv-head (so every K/V
// tile in shared memory feeds two 128x128 score tiles), looping over the key
// tiles of the band [i0 - W + 1, i0 + 127]; key tiles wholly outside the band
// are never loaded, and the mask is evaluated only on tiles the band edge or
// the diagonal cuts.
//
// Warp roles (16 warps):
//   warps 0-3   softmax of head slot 0 (thread = query row)
//   warps 4-7   softmax of head slot 1
//   warps 8-11  Q rotation at start, O rescaling ("correction"), epilogue
//   warp 12     tcgen05.mma issuer (one thread)
//   warp 13     TMA producer (one thread)
//   warps 14-15 idle
// Tensor memory (512 columns): S0 [0,128) S1 [128,256) O0 [256,384)
// O1 [384,512); P (bf16, two per column) overwrites the first 64 columns of
// its S tile once the softmax has read S.
//
// Pipeline per key tile j and head slot s:
//   MMA:     S_s = Q_s K_j^T            -> s_full[s]
//   softmax: m, alpha, P_s -> TMEM      -> alpha_full[s], p_full[s]
//   correct: wait PV_s(j-1), O_s *= alpha (skipped when alpha == 1 for the
//            whole warp)                -> o_ready[s]
//   MMA:     O_s += P_s V_j             -> pv_done[s]
// The max used for the exponentials only moves when the new row max exceeds
// it by more than 8 (log2 units), so most tiles need no O rescale; exp2 of a
// score then stays below 2^8, and the final normalisation by the row sum
// computed with the same max is exact.
#pragma once
#include "swa_internal.cuh"

namespace swa {

namespace prefill_detail {

constexpr int BM = 128;                       // query rows per tile
constexpr int BN = 128;                       // keys per tile
constexpr int NKV = 4;                        // K/V ring buffers
constexpr int kThreads = 512;
constexpr uint32_t kBoxBytes = 128 * 128;     // 128 rows x 64 bf16
constexpr uint32_t kTileBytes = 2 * kBoxBytes;  // 128 rows x 128 bf16
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;     // log2 units

struct PrefillSmem {
  uint8_t q[2][kTileBytes];
  uint8_t kv[NKV][kTileBytes];
  float alpha[2][BM];
  float lsum[2][BM];
  uint64_t q_full[2], q_ready[2];
  uint64_t kv_full[NKV], kv_empty[NKV];
  uint64_t s_full[2], p_full[2], alpha_full[2], o_ready[2], pv_done[2], l_full[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ uint32_t sw128_off(int row, int chunk) {
  return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ void fail(volatile int* abort_flag, int code) {
  record_error(code);
  *abort_flag = 1;
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// Rotate one query row of a Q tile in shared memory (two 64-dim boxes with
// 128-byte swizzle): pairs (k, k + r/2) for k < r/2, cos/sin from the table.
__device__ __forceinline__ void rotate_q_row(uint8_t* tile, int row, int r, const float2* cs) {
  const int half = r / 2;
  if ((half & 7) == 0) {
    for (int c0 = 0; c0 < half / 8; ++c0) {
      const int ea = c0 * 8, eb = ea + half;  // first element of each 8-wide chunk
      uint4* pa = reinterpret_cast<uint4*>(tile + (ea >> 6) * kBoxBytes + sw128_off(row, (ea & 63) >> 3));
      uint4* pb = reinterpret_cast<uint4*>(tile + (eb >> 6) * kBoxBytes + sw128_off(row, (eb & 63) >> 3));
      uint4 A = *pa, Bv = *pb;
      uint32_t* a32 = reinterpret_cast<uint32_t*>(&A);
      uint32_t* b32 = reinterpret_cast<uint32_t*>(&Bv);
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float2 cs0 = cs[ea + 2 * w], cs1 = cs[ea + 2 * w + 1];
        const float x0 = bf16_lo(a32[w]), x1 = bf16_hi(a32[w]);
        const float y0 = bf16_lo(b32[w]), y1 = bf16_hi(b32[w]);
        a32[w] = pack_bf16x2(x0 * cs0.x - y0 * cs0.y, x1 * cs1.x - y1 * cs1.y);
        b32[w] = pack_bf16x2(y0 * cs0.x + x0 * cs0.y, y1 * cs1.x + x1 * cs1.y);
      }
      *pa = A;
      *pb = Bv;
    }
  } else {
    for (int k = 0; k < half; ++k) {
      const int ea = k, eb = k + half;
      uint16_t* pa = reinterpret_cast<uint16_t*>(tile + (ea >> 6) * kBoxBytes + sw128_off(row, (ea & 63) >> 3)) +
                     (ea & 7);
      uint16_t* pb = reinterpret_cast<uint16_t*>(tile + (eb >> 6) * kBoxBytes + sw128_off(row, (eb & 63) >> 3)) +
                     (eb & 7);
      const float x = __uint_as_float((uint32_t)*pa << 16), y = __uint_as_float((uint32_t)*pb << 16);
      const float2 c = cs[k];
      *pa = __bfloat16_as_ushort(__float2bfloat16_rn(x * c.x - y * c.y));
      *pb = __bfloat16_as_ushort(__float2bfloat16_rn(y * c.x + x * c.y));
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const PrefillArgs a, const __grid_constant__ CUtensorMap q_map,
                   const __grid_constant__ CUtensorMap k_map, const __grid_constant__ CUtensorMap v_map) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  PrefillSmem& sm =
      *reinterpret_cast<PrefillSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- which tile: heaviest query tiles (latest rows) first
  const int per_qt = a.n_head_pairs * a.Hkv * a.B;
  const int qt = a.n_q_tiles - 1 - (int)(blockIdx.x / per_qt);
  int rem = (int)(blockIdx.x % per_qt);
  const int hp = rem % a.n_head_pairs;
  rem /= a.n_head_pairs;
  const int kvh = rem % a.Hkv;
  const int b = rem / a.Hkv;
  const int head[2] = {kvh * a.G + 2 * hp, kvh * a.G + min(2 * hp + 1, a.G - 1)};
  const bool store1 = 2 * hp + 1 < a.G;
  const int i0 = qt * BM;
  const int row_last = min(i0 + BM - 1, a.S - 1);
  const int key_lo = a.window > 0 ? max(0, i0 - a.window + 1) : 0;
  const int kt_lo = key_lo / BN, kt_hi = row_last / BN;
  const int n_kv = kt_hi - kt_lo + 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.q_full[s], 1);
      mbar_init(&sm.q_ready[s], BM);
      mbar_init(&sm.s_full[s], 1);
      mbar_init(&sm.p_full[s], BM);
      mbar_init(&sm.alpha_full[s], BM);
      mbar_init(&sm.o_ready[s], BM);
      mbar_init(&sm.pv_done[s], 1);
      mbar_init(&sm.l_full[s], BM);
    }
    for (int i = 0; i < NKV; ++i) {
      mbar_init(&sm.kv_full[i], 1);
      mbar_init(&sm.kv_empty[i], 1);
    }
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort_flag;

  if (warp == 13) {
    // ============================================================ producer
    if (lane == 0) {
      prefetch_tensormap(&q_map);
      prefetch_tensormap(&k_map);
      prefetch_tensormap(&v_map);
      for (int s = 0; s < 2; ++s) {
        mbar_arrive_expect_tx(&sm.q_full[s], kTileBytes);
        tma_load_4d(sm.q[s], &q_map, &sm.q_full[s], 0, head[s], i0, b);
        tma_load_4d(sm.q[s] + kBoxBytes, &q_map, &sm.q_full[s], 64, head[s], i0, b);
      }
      int issued = 0;
      for (int t = 0; t < 2 * n_kv; ++t) {
        const int buf = t % NKV, u = t / NKV;
        if (u > 0 && !mbar_wait(&sm.kv_empty[buf], (u - 1) & 1, abort_flag)) {
          fail(abort_flag, kErrPrefill + 1);
          break;
        }
        mbar_arrive_expect_tx(&sm.kv_full[buf], kTileBytes);
        const int key0 = (kt_lo + (t >> 1)) * BN;
        const CUtensorMap* map = (t & 1) ? &v_map : &k_map;
        tma_load_4d(sm.kv[buf], map, &sm.kv_full[buf], 0, kvh, key0, b);
        tma_load_4d(sm.kv[buf] + kBoxBytes, map, &sm.kv_full[buf], 64, kvh, key0, b);
        issued = t + 1;
      }
      if (*abort_flag) {
        for (int s = 0; s < 2; ++s) mbar_wait(&sm.q_full[s], 0, nullptr, 200000000ull);
        for (int t = issued > NKV ? issued - NKV : 0; t < issued; ++t)
          mbar_wait(&sm.kv_full[t % NKV], (t / NKV) & 1, nullptr, 200000000ull);
      }
    }
  } else if (warp == 12) {
    // ============================================================ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_qk = idesc_bf16_f32(BM, BN, false, false);
      const uint32_t idesc_pv = idesc_bf16_f32(BM, 128, false, true);
      const uint32_t qa[2] = {smem_u32(sm.q[0]), smem_u32(sm.q[1])};
      bool ok = mbar_wait(&sm.q_ready[0], 0, abort_flag) && mbar_wait(&sm.q_ready[1], 0, abort_flag);
      if (!ok) fail(abort_flag, kErrPrefill + 2);
      tc_fence_after();

      auto wait_kv = [&](int t) -> bool {
        if (!mbar_wait(&sm.kv_full[t % NKV], (t / NKV) & 1, abort_flag)) {
          fail(abort_flag, kErrPrefill + 3);
          return false;
        }
        tc_fence_after();
        return true;
      };
      auto issue_qk = [&](int s, uint32_t kb) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kBoxBytes + (kk & 3) * 32;
          umma_ss(tmem + s * 128, sw128_desc(qa[s] + off, 16, 1024), sw128_desc(kb + off, 16, 1024), idesc_qk,
                  kk > 0);
        }
        umma_commit(&sm.s_full[s]);
      };
      auto issue_pv = [&](int s, uint32_t vb, bool acc) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          umma_ts(tmem + 256 + s * 128, tmem + s * 128 + kk * 8, sw128_desc(vb + kk * 2048, kBoxBytes, 1024),
                  idesc_pv, (acc || kk > 0) ? 1u : 0u);
        }
        umma_commit(&sm.pv_done[s]);
      };
      auto wait_pv_inputs = [&](int s, int j) -> bool {
        if (!mbar_wait(&sm.p_full[s], j & 1, abort_flag) || !mbar_wait(&sm.o_ready[s], j & 1, abort_flag)) {
          fail(abort_flag, kErrPrefill + 4);
          return false;
        }
        tc_fence_after();
        return true;
      };

      if (ok && wait_kv(0)) {
        const uint32_t kb0 = smem_u32(sm.kv[0]);
        issue_qk(0, kb0);
        issue_qk(1, kb0);
        umma_commit(&sm.kv_empty[0]);
        for (int j = 0; j < n_kv; ++j) {
          const int tv = 2 * j + 1, tk = 2 * j + 2;
          if (!wait_kv(tv)) break;
          const uint32_t vb = smem_u32(sm.kv[tv % NKV]);
          const uint32_t kb = smem_u32(sm.kv[tk % NKV]);
          const bool more = j + 1 < n_kv;
          if (!wait_pv_inputs(0, j)) break;
          issue_pv(0, vb, j > 0);
          if (more) {
            if (!wait_kv(tk)) break;
            issue_qk(0, kb);
          }
          if (!wait_pv_inputs(1, j)) break;
          issue_pv(1, vb, j > 0);
          umma_commit(&sm.kv_empty[tv % NKV]);
          if (more) {
            issue_qk(1, kb);
            umma_commit(&sm.kv_empty[tk % NKV]);
          }
        }
      }
      // all MMAs issued by this thread complete before the CTA moves on
      umma_commit(&sm.drain);
      mbar_wait(&sm.drain, 0, nullptr, 200000000ull);
    }
  } else if (warp < 8) {
    // ============================================================ softmax
    const int s = warp >> 2;
    const int row = threadIdx.x & (BM - 1);
    const int i = i0 + row;
    const uint32_t taddr = tmem + ((uint32_t)((warp & 3) * 32) << 16) + s * 128;
    const float c = a.scale_log2;
    float m = -INFINITY, l = 0.f;
    for (int j = 0; j < n_kv; ++j) {
      const int key0 = (kt_lo + j) * BN;
      const bool got = mbar_wait(&sm.s_full[s], j & 1, abort_flag);
      __syncwarp();  // tcgen05.ld below is warp-collective
      if (!__all_sync(0xffffffffu, got)) {
        fail(abort_flag, kErrPrefill + 5);
        break;
      }
      tc_fence_after();
      const bool full_tile = key0 + BN - 1 <= i0 && (a.window < 0 || key0 >= i0 + BM - 1 - a.window + 1);
      // visible keys of this row inside the tile: [lo, hi] (tile-relative)
      const int hi = i - key0;
      const int lo = a.window < 0 ? 0 : i - a.window + 1 - key0;
      // pass 1: row max
      float mx = -INFINITY;
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        uint32_t v[32];
        tmem_ld32(taddr + q4 * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int col = q4 * 32 + e;
          float x = __uint_as_float(v[e]);
          if (!full_tile && (col > hi || col < lo)) x = -INFINITY;
          mx = fmaxf(mx, x);
        }
      }
      const float mt = mx * c;
      const float m_use = (mt - m > kRescaleThreshold) ? mt : m;  // m = -inf: always take mt
      const float m_safe = m_use == -INFINITY ? 0.f : m_use;
      const float alpha = fast_exp2(m - m_safe);
      sm.alpha[s][row] = alpha;
      mbar_arrive(&sm.alpha_full[s]);
      // pass 2: P = exp2(c S - m), row sum, bf16 P back into TMEM
      float sum = 0.f;
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        uint32_t v[32];
        tmem_ld32(taddr + q4 * 32, v);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const int col = q4 * 32 + e;
          float p0 = fast_exp2(__uint_as_float(v[e]) * c - m_safe);
          float p1 = fast_exp2(__uint_as_float(v[e + 1]) * c - m_safe);
          if (!full_tile) {
            if (col > hi || col < lo) p0 = 0.f;
            if (col + 1 > hi || col + 1 < lo) p1 = 0.f;
          }
          sum += p0 + p1;
          pk[e >> 1] = pack_bf16x2(p0, p1);
        }
        tmem_st16(taddr + q4 * 16, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.p_full[s]);
      l = l * alpha + sum;
      m = m_use;
    }
    sm.lsum[s][row] = l;
    mbar_arrive(&sm.l_full[s]);
  } else if (warp < 12) {
    // ============================================================ correction
    const int row = threadIdx.x & (BM - 1);
    const int i = i0 + row;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    // Q rotation in shared memory (both head slots)
    for (int s = 0; s < 2; ++s) {
      if (!mbar_wait(&sm.q_full[s], 0, abort_flag)) {
        fail(abort_flag, kErrPrefill + 6);
        break;
      }
      if (a.rotary_dim > 0 && i < a.S)
        rotate_q_row(sm.q[s], row, a.rotary_dim, a.table + (size_t)i * (a.rotary_dim / 2));
      fence_proxy_async_smem();
      mbar_arrive(&sm.q_ready[s]);
    }
    bool ok = !*abort_flag;
    for (int j = 0; j < n_kv && ok; ++j) {
      for (int s = 0; s < 2 && ok; ++s) {
        const bool got_a = mbar_wait(&sm.alpha_full[s], j & 1, abort_flag);
        if (!__all_sync(0xffffffffu, got_a)) {
          fail(abort_flag, kErrPrefill + 7);
          ok = false;
          break;
        }
        const float alpha = sm.alpha[s][row];
        if (j > 0) {
          const bool got_pv = mbar_wait(&sm.pv_done[s], (j - 1) & 1, abort_flag);
          if (!__all_sync(0xffffffffu, got_pv)) {
            fail(abort_flag, kErrPrefill + 8);
            ok = false;
            break;
          }
          tc_fence_after();
          if (__any_sync(0xffffffffu, alpha != 1.f)) {
            const uint32_t oaddr = tmem + lane_off + 256 + s * 128;
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              uint32_t v[32];
              tmem_ld32(oaddr + q4 * 32, v);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
              tmem_st32(oaddr + q4 * 32, v);
            }
            tmem_wait_st();
          }
        }
        tc_fence_before();
        mbar_arrive(&sm.o_ready[s]);
      }
    }
    // epilogue: out = O / l * sigmoid(gate)
    for (int s = 0; s < 2 && ok; ++s) {
      const bool got_o = mbar_wait(&sm.pv_done[s], (n_kv - 1) & 1, abort_flag) &&
                         mbar_wait(&sm.l_full[s], 0, abort_flag);
      if (!__all_sync(0xffffffffu, got_o)) {
        fail(abort_flag, kErrPrefill + 9);
        break;
      }
      tc_fence_after();
      const float l = sm.lsum[s][row];
      const bool live = i < a.S && (s == 0 || store1);
      float g = 1.f;
      if (a.gate && live) g = 1.f / (1.f + __expf(-a.gate[((size_t)b * a.S + i) * a.Hq + head[s]]));
      const float f = g / l;
      uint16_t* dst = a.out + (((size_t)b * a.S + (live ? i : 0)) * a.Hq + head[s]) * 128;
      const uint32_t oaddr = tmem + lane_off + 256 + s * 128;
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        uint32_t v[32];
        tmem_ld32(oaddr + q4 * 32, v);
        tmem_wait_ld();
        if (live) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + q4 * 32);
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            uint4 u;
            u.x = pack_bf16x2(__uint_as_float(v[8 * w + 0]) * f, __uint_as_float(v[8 * w + 1]) * f);
            u.y = pack_bf16x2(__uint_as_float(v[8 * w + 2]) * f, __uint_as_float(v[8 * w + 3]) * f);
            u.z = pack_bf16x2(__uint_as_float(v[8 * w + 4]) * f, __uint_as_float(v[8 * w + 5]) * f);
            u.w = pack_bf16x2(__uint_as_float(v[8 * w + 6]) * f, __uint_as_float(v[8 * w + 7]) * f);
            d4[w] = u;
          }
        }
      }
    }
  }
  // warps 14-15 (and the idle lanes of 12-13) fall through

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace prefill_detail

cudaError_t launch_prefill(const PrefillArgs& a, const CUtensorMap& q_map, const CUtensorMap& k_map,
                           const CUtensorMap& v_map, cudaStream_t stream) {
  using namespace prefill_detail;
  const long long n_cta = (long long)a.n_q_tiles * a.n_head_pairs * a.Hkv * a.B;
  if (n_cta == 0) return cudaSuccess;
  if (n_cta > 0x7FFFFFFFll) return cudaErrorInvalidConfiguration;
  const size_t smem = sizeof(PrefillSmem) + 1024;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  prefill_kernel<<<(unsigned)n_cta, kThreads, smem, stream>>>(a, q_map, k_map, v_map);
  return cudaGetLastError();
}

}  // namespace swa
