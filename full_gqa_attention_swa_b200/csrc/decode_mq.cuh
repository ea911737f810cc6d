// Multi-query decode on the tensor cores: T new tokens of every sequence
// attend in one call, each through its own band.  The "Step-3.7-Flash" spec
// card's architecture notes list three extra multi-token-prediction (MTP)
// layers that speed up decoding; the tokens they propose are checked this
// way.  The band and the cache rule are the "Step-3.7-Flash-oQ3e" explainer's
// section 2.2 (a sliding layer keeps the last W tokens; query i sees keys
// i - W < j <= i), the gate its section 2.3.
//
// The cache holds the L0 = L - T earlier tokens (ring slot p mod W, or slot
// p); the new tokens' rotated keys and values come separately, so checking
// drafts never overwrites ring slots an earlier query still needs.  Query t
// sits at position L0 + t.  On a ring, dist(s) = (s - n - 1) mod W numbers the
// slots from the oldest (n = slot of position L0 - 1); query t sees exactly the
// slots with dist > t, and new key j iff t - W < j <= t.
//
// Work split: one CTA per (sequence, kv-head, split of the cache).  The T * G
// (query, head) rows of the kv-head (<= 64) are the M dimension of
// tcgen05.mma (M = 128, rows past T * G are zero), so a key block costs the
// tensor core a handful of instructions: S = Q K^T (N = 64 keys) into tensor
// memory, the softmax (thread = row) writes P (bf16) over S, and
// O += P V reads P from tensor memory.  S is double-buffered (two 64-column
// tiles), so the QK^T of block j + 1 overlaps the softmax of block j.  K and V
// stream through separate TMA rings (three and two 64-key stages).  At 96 KB
// of shared memory and 256 tensor-memory columns a CTA, two CTAs share an SM.
// The last split also runs one 16-key block of the new tokens.
#pragma once
#include "swa_internal.cuh"

namespace swa {

namespace decode_mq_detail {

constexpr int KB = 64;                           // keys per cache block
constexpr int kNewRows = 16;                     // new-token block (T <= 16)
constexpr int kKStages = 3, kVStages = 2;
constexpr uint32_t kBoxBytes = KB * 128;         // 64 rows x 64 bf16
constexpr uint32_t kBlockBytes = 2 * kBoxBytes;  // 64 keys x 128 dims
constexpr uint32_t kNewBoxBytes = kNewRows * 128;
constexpr int kThreads = 160;                    // softmax warps 0-1, K producer 2, issuer 3, V producer 4
constexpr uint32_t kTmemCols = 256;              // S0 [0,64) S1 [64,128) O [128,256)
static_assert(kNewRows == kDecodeMqMaxT, "one block holds every new token");
static_assert(kDecodeMqMaxRows <= 64, "rows fit the two softmax warps");

struct Smem {
  uint8_t q[2 * kBoxBytes];                  // rows (t, g) < 64 of both 64-dim halves
  uint8_t k[kKStages][kBlockBytes];
  uint8_t v[kVStages][kBlockBytes];
  uint64_t q_full;
  uint64_t k_full[kKStages], k_empty[kKStages];
  uint64_t v_full[kVStages], v_empty[kVStages];
  uint64_t s_full[2], p_full[2], pv_done[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

// Wait that sleeps between tests, for roles whose waits are not on the
// critical path (the TMA producers): a tight polling loop takes issue slots
// from the softmax warps that share its sub-partition.
__device__ __forceinline__ bool mbar_wait_sleep(uint64_t* bar, uint32_t parity, volatile int* abort, uint32_t ns) {
  if (mbar_test(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    __nanosleep(ns);
    if (mbar_test(bar, parity)) return true;
    if ((it & 15u) == 0) {
      if (abort != nullptr && *abort) return false;
      if (globaltimer() - t0 > kWaitLimitNs) return false;
    }
  }
}

__device__ __forceinline__ uint32_t sw128_off(int row, int chunk) {
  return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ float sigmoidf_(float g) { return 1.f / (1.f + __expf(-g)); }

__device__ __forceinline__ void fail(volatile int* abort_flag, int code) {
  record_error(code);
  *abort_flag = 1;
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  const bool got = mbar_wait(bar, parity, abort_flag);
  return __all_sync(0xffffffffu, got);
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t* r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}

// grid (max_splits, Hkv, B)
__global__ void __launch_bounds__(kThreads, 2)
    decode_mq_kernel(const DecodeMqArgs a, const __grid_constant__ CUtensorMap q_map,
                     const __grid_constant__ CUtensorMap k_map, const __grid_constant__ CUtensorMap v_map,
                     const __grid_constant__ CUtensorMap kn_map, const __grid_constant__ CUtensorMap vn_map) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  allow_dependent_launch();
  grid_dependency_wait();
  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int T = a.T, G = a.G, n_rows = T * G;
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
  const int n_cb = k_end > k_begin ? (k_end - k_begin + KB - 1) / KB : 0;  // cache blocks
  const bool has_new = split == n_split - 1;
  const int n_tot = n_cb + (has_new ? 1 : 0);  // >= 1
  const int newest = (ring && L0 > 0) ? (L0 - 1) % a.window : 0;  // ring slot of position L0 - 1

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.k_empty[s], 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.s_full[s], 1);
      mbar_init(&sm.p_full[s], 2);  // one arrival per softmax warp
      mbar_init(&sm.pv_done[s], 1);
    }
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  // rows n_rows .. 63 of Q stay zero (the TMA box writes only the first n_rows)
  for (int i = threadIdx.x; i < (int)(2 * kBoxBytes / 16); i += kThreads)
    reinterpret_cast<uint4*>(sm.q)[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  if (warp == 0) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort_flag;
  const int row3 = b * a.Hkv + kvh;

  if (warp == 2) {
    // ---------------------------------------------------- Q and K producer
    if (lane == 0) {
      prefetch_tensormap(&q_map);
      prefetch_tensormap(&k_map);
      mbar_arrive_expect_tx(&sm.q_full, 2u * 128u * (uint32_t)n_rows);
      tma_load_4d(sm.q, &q_map, &sm.q_full, 0, kvh * G, 0, b);
      tma_load_4d(sm.q + kBoxBytes, &q_map, &sm.q_full, 64, kvh * G, 0, b);
      int issued = 0;
      for (int j = 0; j < n_tot; ++j) {
        const int st = j % kKStages;
        if (j >= kKStages && !mbar_wait_sleep(&sm.k_empty[st], (j / kKStages - 1) & 1, abort_flag, 256)) {
          fail(abort_flag, kErrDecodeMq + 1);
          break;
        }
        if (j < n_cb) {
          const int key0 = k_begin + j * KB;
          mbar_arrive_expect_tx(&sm.k_full[st], kBlockBytes);
          tma_load_3d(sm.k[st], &k_map, &sm.k_full[st], 0, key0, row3);
          tma_load_3d(sm.k[st] + kBoxBytes, &k_map, &sm.k_full[st], 64, key0, row3);
        } else {
          mbar_arrive_expect_tx(&sm.k_full[st], 2 * kNewBoxBytes);
          tma_load_4d(sm.k[st], &kn_map, &sm.k_full[st], 0, kvh, 0, b);
          tma_load_4d(sm.k[st] + kBoxBytes, &kn_map, &sm.k_full[st], 64, kvh, 0, b);
        }
        issued = j + 1;
      }
      if (*abort_flag) {
        mbar_wait(&sm.q_full, 0, nullptr, 200000000ull);
        for (int j = issued > kKStages ? issued - kKStages : 0; j < issued; ++j)
          mbar_wait(&sm.k_full[j % kKStages], (j / kKStages) & 1, nullptr, 200000000ull);
      }
    }
  } else if (warp == 4) {
    // ---------------------------------------------------------- V producer
    if (lane == 0) {
      prefetch_tensormap(&v_map);
      int issued = 0;
      for (int j = 0; j < n_tot; ++j) {
        const int st = j % kVStages;
        if (j >= kVStages && !mbar_wait_sleep(&sm.v_empty[st], (j / kVStages - 1) & 1, abort_flag, 256)) {
          fail(abort_flag, kErrDecodeMq + 5);
          break;
        }
        if (j < n_cb) {
          const int key0 = k_begin + j * KB;
          mbar_arrive_expect_tx(&sm.v_full[st], kBlockBytes);
          tma_load_3d(sm.v[st], &v_map, &sm.v_full[st], 0, key0, row3);
          tma_load_3d(sm.v[st] + kBoxBytes, &v_map, &sm.v_full[st], 64, key0, row3);
        } else {
          mbar_arrive_expect_tx(&sm.v_full[st], 2 * kNewBoxBytes);
          tma_load_4d(sm.v[st], &vn_map, &sm.v_full[st], 0, kvh, 0, b);
          tma_load_4d(sm.v[st] + kBoxBytes, &vn_map, &sm.v_full[st], 64, kvh, 0, b);
        }
        issued = j + 1;
      }
      if (*abort_flag)
        for (int j = issued > kVStages ? issued - kVStages : 0; j < issued; ++j)
          mbar_wait(&sm.v_full[j % kVStages], (j / kVStages) & 1, nullptr, 200000000ull);
    }
  } else if (warp == 3) {
    // ----------------------------------------------------------- MMA issuer
    // QK^T(j) into S[j & 1], then P(j - 1).V: the QK^T of a block overlaps the
    // softmax of the previous one.  QK^T(j) overwrites the columns of P(j - 2)
    // only after P(j - 2).V, issued before it, has read them.
    if (lane == 0) {
      const uint64_t qd = sw128_desc(smem_u32(sm.q), 16, 1024);
      const uint64_t kd = sw128_desc(smem_u32(sm.k[0]), 16, 1024);
      const uint64_t vd = sw128_desc(smem_u32(sm.v[0]), kBoxBytes, 1024);
      const uint32_t idesc_qk = idesc_bf16_f32(128, KB, false, false);
      const uint32_t idesc_qk_new = idesc_bf16_f32(128, kNewRows, false, false);
      const uint32_t idesc_pv = idesc_bf16_f32(128, 128, false, true);
      bool ok = mbar_wait(&sm.q_full, 0, abort_flag);
      int issued_pv = 0;
      auto pv = [&](int x) -> bool {
        if (!mbar_wait(&sm.p_full[x & 1], (x >> 1) & 1, abort_flag) ||
            !mbar_wait(&sm.v_full[x % kVStages], (x / kVStages) & 1, abort_flag))
          return false;
        tc_fence_after();
        const uint32_t b0 = (uint32_t)vd + (uint32_t)(((x % kVStages) * kBlockBytes) >> 4);
        const int n_k16 = x < n_cb ? KB / 16 : 1;
        for (int kk = 0; kk < n_k16; ++kk)
          umma_ts_lh(tmem + 128, tmem + (x & 1) * 64 + kk * 8, b0 + (uint32_t)((kk * 2048) >> 4),
                     (uint32_t)(vd >> 32), idesc_pv, (x > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&sm.v_empty[x % kVStages]);
        umma_commit(&sm.pv_done[x & 1]);
        issued_pv = x + 1;
        return true;
      };
      for (int j = 0; j < n_tot && ok; ++j) {
        ok = mbar_wait(&sm.k_full[j % kKStages], (j / kKStages) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        const uint32_t b0 = (uint32_t)kd + (uint32_t)(((j % kKStages) * kBlockBytes) >> 4);
        const uint32_t idesc = j < n_cb ? idesc_qk : idesc_qk_new;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (uint32_t)((((kk >> 2) * kBoxBytes) + (kk & 3) * 32) >> 4);
          umma_ss_lh(tmem + (j & 1) * 64, (uint32_t)qd + off, (uint32_t)(qd >> 32), b0 + off, (uint32_t)(kd >> 32),
                     idesc, kk > 0);
        }
        umma_commit(&sm.s_full[j & 1]);
        umma_commit(&sm.k_empty[j % kKStages]);
        if (j > 0) ok = pv(j - 1);
      }
      if (ok) ok = pv(n_tot - 1);
      if (!ok) fail(abort_flag, kErrDecodeMq + 6);
      (void)issued_pv;
      // every MMA of this thread completes before the CTA moves on
      umma_commit(&sm.drain);
      mbar_wait(&sm.drain, 0, nullptr, 200000000ull);
    }
  } else if (warp < 2) {
    // ------------------------------------------------ softmax (thread = row)
    const int r = threadIdx.x;  // 0..63
    const bool valid = r < n_rows;
    const int t = valid ? r / G : 0;
    const int hq = kvh * G + (valid ? r % G : 0);
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const float c = a.scale_log2;
    const int W = a.window;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_tot; ++j) {
      const bool is_new = j >= n_cb;
      const int key0 = k_begin + j * KB;
      const int live = is_new ? T : k_end - key0;  // keys of the block that exist
      if (!warp_wait(&sm.s_full[j & 1], (j >> 1) & 1, abort_flag)) {
        fail(abort_flag, kErrDecodeMq + 2);
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t s_addr = tmem + lane_base + (j & 1) * 64;
      uint32_t v[64];
      if (!is_new) {
        tmem_ld32(s_addr, *reinterpret_cast<uint32_t(*)[32]>(v));
        tmem_ld32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
      } else {
        tmem_ld16(s_addr, *reinterpret_cast<uint32_t(*)[16]>(v));
      }
      tmem_wait_ld();
      // A cache block needs per-key masks only when it is ragged or, on a
      // ring, holds one of the T oldest slots (ring distance < T); the rows past
      // T * G read zero queries and need none.  Scores are kept unscaled
      // (raw dot products); the scale goes into the exponent.
      const int dbase = key0 - newest - 1;  // ring distance of key 0 of the block, unwrapped
      const int d0 = dbase < 0 ? dbase + W : dbase;
      const bool masked = is_new || live < KB || (ring && (d0 < T || (dbase < 0 && dbase + KB > 0)));
      float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      if (is_new) {
#pragma unroll
        for (int e = 0; e < kNewRows; ++e) {
          const bool vis = e < live && e <= t && (!ring || e > t - W);
          if (!vis) v[e] = __float_as_uint(-INFINITY);
          mx[e & 3] = fmaxf(mx[e & 3], __uint_as_float(v[e]));
        }
      } else if (masked) {
#pragma unroll
        for (int e = 0; e < KB; ++e) {
          int dd = dbase + e;
          dd += dd < 0 ? W : 0;
          const bool vis = e < live && (!ring || dd > t);
          if (!vis) v[e] = __float_as_uint(-INFINITY);
          mx[e & 3] = fmaxf(mx[e & 3], __uint_as_float(v[e]));
        }
      } else {
#pragma unroll
        for (int e = 0; e < KB; e += 2)
          mx[(e >> 1) & 3] = fmax3(mx[(e >> 1) & 3], __uint_as_float(v[e]), __uint_as_float(v[e + 1]));
      }
      const float mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * c;
      const float m_use = (mt - m > 8.f) ? mt : m;  // lazy: the max moves only by more than 8
      const float m_safe = m_use == -INFINITY ? 0.f : m_use;
      const float alpha = fast_exp2(m - m_safe);
      float sum = 0.f;
      uint32_t pk[32];
      if (is_new) {
#pragma unroll
        for (int e = 0; e < kNewRows; e += 2) {
          const float p0 = fast_exp2(fmaf(__uint_as_float(v[e]), c, -m_safe));
          const float p1 = fast_exp2(fmaf(__uint_as_float(v[e + 1]), c, -m_safe));
          sum += p0 + p1;
          pk[e >> 1] = pack_bf16x2(p0, p1);
        }
      } else {
        const uint64_t cc = f2_pack(c, c), mm = f2_pack(-m_safe, -m_safe);
        uint64_t s2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int e = 0; e < KB; e += 2) {
          const uint64_t y = f2_fma(f2_pack(__uint_as_float(v[e]), __uint_as_float(v[e + 1])), cc, mm);
          float y0, y1;
          f2_unpack(y, y0, y1);
          const float p0 = fast_exp2(y0), p1 = fast_exp2(y1);
          s2[(e >> 1) & 3] = f2_add(s2[(e >> 1) & 3], f2_pack(p0, p1));
          pk[e >> 1] = pack_bf16x2(p0, p1);
        }
        float a0, a1;
        f2_unpack(f2_add(f2_add(s2[0], s2[1]), f2_add(s2[2], s2[3])), a0, a1);
        sum = a0 + a1;
      }
      // P over the S columns it came from
      if (!is_new) {
        tmem_st32(s_addr, *reinterpret_cast<const uint32_t(*)[32]>(pk));
      } else {
        tmem_st8(s_addr, pk);
      }
      // keys no row sees (past the live end; a full ring's oldest slot) may
      // hold NaN: zero their V rows before P.V, which multiplies them by 0
      const int dead = (ring && L0 >= W && !is_new) ? (newest + 1) % W - key0 : -1;
      const bool ragged = !is_new && live < KB;
      const bool dead_in = (unsigned)dead < (unsigned)KB;
      if (ragged || dead_in) {
        if (!warp_wait(&sm.v_full[j % kVStages], (j / kVStages) & 1, abort_flag)) {
          fail(abort_flag, kErrDecodeMq + 7);
          ok = false;
          break;
        }
        uint8_t* vst = sm.v[j % kVStages];
        // thread r zeroes key row r (64 rows, 64 threads)
        if (r >= live || r == dead) {
#pragma unroll
          for (int ch = 0; ch < 16; ++ch)
            *reinterpret_cast<uint4*>(vst + (ch >> 3) * kBoxBytes + sw128_off(r, ch & 7)) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
      }
      // O holds blocks 0..j-1: bring it to the new max before P(j).V adds to it
      // (a row that has seen no key yet holds O = 0 and needs nothing)
      if (j > 0 && __any_sync(0xffffffffu, valid && m != -INFINITY && alpha != 1.f)) {
        if (!warp_wait(&sm.pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag)) {
          fail(abort_flag, kErrDecodeMq + 8);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t o_addr = tmem + lane_base + 128;
#pragma unroll 1
        for (int q4 = 0; q4 < 4; ++q4) {
          uint32_t o[32];
          tmem_ld32(o_addr + q4 * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(o_addr + q4 * 32, o);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.p_full[j & 1]);
      l = l * alpha + sum;
      m = m_use;
    }
    // ---- result: the last P.V complete, then O of this row
    if (ok && warp_wait(&sm.pv_done[(n_tot - 1) & 1], ((n_tot - 1) >> 1) & 1, abort_flag)) {
      tc_fence_after();
      const uint32_t o_addr = tmem + lane_base + 128;
      const size_t row = ((size_t)b * T + t) * a.Hq + hq;
      const float f = (a.max_splits == 1) ? (a.gate ? sigmoidf_(a.gate[row]) : 1.f) / l : 1.f;
#pragma unroll 1
      for (int q4 = 0; q4 < 4; ++q4) {
        uint32_t o[32];
        tmem_ld32(o_addr + q4 * 32, o);
        tmem_wait_ld();
        if (valid) {
          if (a.max_splits == 1) {
            uint4* dst = reinterpret_cast<uint4*>(a.out + row * kHeadDim) + q4 * 4;
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4)
              dst[c4] = make_uint4(pack_bf16x2(__uint_as_float(o[8 * c4]) * f, __uint_as_float(o[8 * c4 + 1]) * f),
                                   pack_bf16x2(__uint_as_float(o[8 * c4 + 2]) * f, __uint_as_float(o[8 * c4 + 3]) * f),
                                   pack_bf16x2(__uint_as_float(o[8 * c4 + 4]) * f, __uint_as_float(o[8 * c4 + 5]) * f),
                                   pack_bf16x2(__uint_as_float(o[8 * c4 + 6]) * f, __uint_as_float(o[8 * c4 + 7]) * f));
          } else {
            const size_t slot = row * a.max_splits + split;
            float4* dst = reinterpret_cast<float4*>(a.part_o + slot * kHeadDim) + q4 * 8;
#pragma unroll
            for (int c4 = 0; c4 < 8; ++c4)
              dst[c4] = make_float4(__uint_as_float(o[4 * c4]), __uint_as_float(o[4 * c4 + 1]),
                                    __uint_as_float(o[4 * c4 + 2]), __uint_as_float(o[4 * c4 + 3]));
            if (q4 == 0) a.part_ml[slot] = make_float2(m, l);
          }
        }
      }
    } else if (ok) {
      fail(abort_flag, kErrDecodeMq + 9);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
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

}  // namespace decode_mq_detail

cudaError_t launch_decode_mq(const DecodeMqArgs& a, const CUtensorMap& q_map, const CUtensorMap& k_map,
                             const CUtensorMap& v_map, const CUtensorMap& kn_map, const CUtensorMap& vn_map,
                             cudaStream_t stream) {
  using namespace decode_mq_detail;
  if (a.B == 0) return cudaSuccess;
  const size_t smem = sizeof(Smem) + 1024;
  static DeviceOnce setup;
  cudaError_t e = device_once(setup, [&](int, int*) {
    return cudaFuncSetAttribute(decode_mq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  });
  if (e != cudaSuccess) return e;
  e = launch_kernel(true, decode_mq_kernel, dim3(a.max_splits, a.Hkv, a.B), dim3(kThreads), smem, stream, a,
                    q_map, k_map, v_map, kn_map, vn_map);
  if (e != cudaSuccess || a.max_splits == 1) return e;
  return launch_kernel(true, decode_mq_combine_kernel, dim3(a.Hq, a.T, a.B), dim3(kHeadDim), 0,
                       stream, a);
}

}  // namespace swa
