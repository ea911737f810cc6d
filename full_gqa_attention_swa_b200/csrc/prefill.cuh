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
// Work unit ("tile"): 128 query rows x two q-heads ("head slots") of the same
// kv-head, so every K/V tile in shared memory feeds two 128x128 score tiles.
// Query row r sits at key-space position i = q_off + r.  A tile loops over
// the key tiles of its band [i0 - W + 1, i0 + 127]; key tiles wholly outside
// the band are never loaded, and the mask is evaluated only on tiles the band
// edge or the diagonal cuts.  The grid is persistent (one CTA per SM); a CTA
// walks tiles blockIdx.x, +gridDim.x, ... with the longest (latest-row) tiles
// first.
//
// Pipeline.  P (bf16) is written by the softmax into the tensor-memory
// columns of the S tile it came from, and P.V reads it from there (A operand
// in tensor memory), so no shared memory holds P.  That leaves room for two
// Q buffers per head slot: the next tile's Q is loaded and rotated while the
// current tile runs, and the first QK^T of the next tile follows the last P.V
// of this one without a gap.  The tensor pipe runs, per head slot s and key
// tile j, the block [O_s += P_s(j) V(j); S_s = Q_s K(j+1)^T], the two slots'
// blocks alternating, so one slot's softmax overlaps the other slot's MMAs.
// The MMAs of one thread execute in issue order, so S_s(j+1) overwrites the
// columns of P_s(j) only after P_s(j).V has read them.
//
// Warp roles (16 warps, registers rebalanced with setmaxnreg):
//   warps 0-3   head slot 0 softmax (thread = query row); rescales its own
//               O row when the running max moves (rare: lazy threshold)
//   warps 4-7   head slot 1 softmax
//   warps 8-11  next tile's Q rotation, then this tile's epilogue
//               (O / l * sigmoid(gate) -> bf16, thread = row, staged in the
//               tile's own Q buffers and written by TMA stores)
//   warp 12     tcgen05.mma issuer (one thread)
//   warp 13     K / V TMA producer (one thread), three-stage ring
//   warp 15     Q TMA producer (one thread)
// Tensor memory (512 columns): S0/P0 [0,128) S1/P1 [128,256) O0 [256,384)
// O1 [384,512).
// The max used for the exponentials only moves when the new row max exceeds
// it by more than 8 (log2 units), so most key tiles need no O rescale; exp2
// of a score then stays below 2^8, and the final normalisation by the row sum
// computed with the same max is exact.
#pragma once
#include "swa_internal.cuh"

namespace swa {

namespace prefill_detail {

constexpr int BM = 128;                         // query rows per tile
constexpr int BN = 128;                         // keys per key tile
constexpr int kKvStages = 3;                    // K / V ring (loads K0 V0 K1 V1 ...)
constexpr int kThreads = 512;
constexpr uint32_t kBoxBytes = 128 * 128;       // 128 rows x 64 bf16
constexpr uint32_t kTileBytes = 2 * kBoxBytes;  // 128 rows x 128 bf16
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;       // log2 units

// setmaxnreg split of the 128 x 512 registers the CTA is launched with
constexpr uint32_t kRegsLaunch = 128;
constexpr uint32_t kRegsSoftmax = 184;
constexpr uint32_t kRegsCorrection = 88;
constexpr uint32_t kRegsOther = 56;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsCorrection + 128 * kRegsOther <= kRegsLaunch * kThreads,
              "register split exceeds the launch allocation");

struct Smem {
  uint8_t q[2][2][kTileBytes];     // [tile parity][head slot]: Q, rotated in place
  uint8_t kv[kKvStages][kTileBytes];
  float lsum[2][2][BM];            // [tile parity][head slot][row]: softmax row sums
  uint64_t q_full[2][2];           // Q of [parity][slot] landed
  uint64_t q_free[2];              // the output staged in Q[parity][*] has been read by its TMA store
  uint64_t q_ready[2];             // both slots' Q rotated (128 arrivals)
  uint64_t kv_full[kKvStages], kv_empty[kKvStages];
  uint64_t s_full[2];              // S_s complete (and every earlier MMA, P_s.V included)
  uint64_t p_full[2];              // P_s written, O_s rescaled (128 arrivals)
  uint64_t o_done[2];              // the tile's last P_s.V complete
  uint64_t o_free[2];              // the epilogue has read O_s (128 arrivals)
  uint64_t o_staged[2];            // the bf16 output of slot s is in shared memory (128 arrivals)
  uint64_t l_full[2][2];           // [parity][slot] row sums written (128 arrivals)
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

struct Tile {
  int qt, kvh, b, h0, h1;
  int r0;  // first query row of the tile (rows of q / out / gate / cos-sin table)
  int i0;  // its key-space position, q_off + r0 (masks and key ranges)
  int kt_lo, n_kv;
  bool store1;
};

// Launch modes: a whole prefill (queries at key positions 0..S-1, K / V as
// [B, S, Hkv, D]), a chunk over an assembled K / V sequence (queries offset by
// q_off), and a chunk over a KV cache [B * Hkv, C, D] read in place.
enum PrefillMode : int { kWhole = 0, kChunkSeq = 1, kChunkCache = 2 };

template <int kMode>
__device__ __forceinline__ Tile decode_tile(const PrefillArgs& a, int t) {
  const int q_off = kMode == kWhole ? 0 : a.q_off;
  Tile T;
  const int per_qt = a.n_head_pairs * a.Hkv * a.B;
  T.qt = a.n_q_tiles - 1 - t / per_qt;  // latest query rows (most keys) first
  int rem = t % per_qt;
  const int hp = rem % a.n_head_pairs;
  rem /= a.n_head_pairs;
  T.kvh = rem % a.Hkv;
  T.b = rem / a.Hkv;
  T.h0 = T.kvh * a.G + 2 * hp;
  T.h1 = T.kvh * a.G + min(2 * hp + 1, a.G - 1);
  T.store1 = 2 * hp + 1 < a.G;
  T.r0 = T.qt * BM;
  T.i0 = q_off + T.r0;
  const int row_last = q_off + min(T.r0 + BM - 1, a.S - 1);
  const int key_lo = a.window > 0 ? max(0, T.i0 - a.window + 1) : 0;
  T.kt_lo = key_lo / BN;
  T.n_kv = row_last / BN - T.kt_lo + 1;
  return T;
}

__device__ __forceinline__ uint32_t sw128_off(int row, int chunk) {
  return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}

// Bits lo .. hi of a 32-bit word (none where hi < lo; bounds outside 0..31
// are clamped).
__device__ __forceinline__ uint32_t chunk_keep(int lo, int hi) {
  const uint32_t to_hi = hi >= 31 ? 0xffffffffu : (hi < 0 ? 0u : (2u << hi) - 1u);  // bits 0 .. hi
  const uint32_t to_lo = lo <= 0 ? 0u : (lo > 31 ? 0xffffffffu : (1u << lo) - 1u);  // bits 0 .. lo - 1
  return to_hi & ~to_lo;
}

__device__ __forceinline__ void fail(volatile int* abort_flag, int code) {
  record_error(code);
  *abort_flag = 1;
}

// Every lane of the warp waits; the result is the same on all lanes so that
// the warp-collective tcgen05 operations that follow run converged.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  const bool got = mbar_wait(bar, parity, abort_flag);
  return __all_sync(0xffffffffu, got);
}

// Rotates dims 8 c0 .. 8 c0 + 7 with their partners 8 c0 + half .. of one
// row of a Q tile in shared memory (two 64-dim boxes, 128-byte swizzle);
// t4[w] holds (cos, sin) of pairs 8 c0 + 2w and 8 c0 + 2w + 1.  Rounding as
// in the RoPE kernels (the partner's product rounded, then one fma), so a
// rotated q equals swa_rope_qk's bit for bit.
__device__ __forceinline__ void rotate_q_chunk(uint8_t* tile, int row, int c0, int half, const float4* t4) {
  const int ea = c0 * 8, eb = ea + half;
  uint4* pa = reinterpret_cast<uint4*>(tile + (ea >> 6) * kBoxBytes + sw128_off(row, (ea & 63) >> 3));
  uint4* pb = reinterpret_cast<uint4*>(tile + (eb >> 6) * kBoxBytes + sw128_off(row, (eb & 63) >> 3));
  uint4 A = *pa, Bv = *pb;
  uint32_t* a32 = reinterpret_cast<uint32_t*>(&A);
  uint32_t* b32 = reinterpret_cast<uint32_t*>(&Bv);
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const float4 t = t4[w];
    const float x0 = bf16_lo(a32[w]), x1 = bf16_hi(a32[w]);
    const float y0 = bf16_lo(b32[w]), y1 = bf16_hi(b32[w]);
    a32[w] = pack_bf16x2(fmaf(x0, t.x, -(y0 * t.y)), fmaf(x1, t.z, -(y1 * t.w)));
    b32[w] = pack_bf16x2(fmaf(y0, t.x, x0 * t.y), fmaf(y1, t.z, x1 * t.w));
  }
  *pa = A;
  *pb = Bv;
}

// Element-wise form for any even r.
__device__ __forceinline__ void rotate_q_row_scalar(uint8_t* tile, int row, int i, int half,
                                                    const float2* __restrict__ table) {
  for (int k = 0; k < half; ++k) {
    const int ea = k, eb = k + half;
    const float2 c = __ldg(table + rope_table_index(i, k, half));
    const uint32_t oa = (ea >> 6) * kBoxBytes + sw128_off(row, (ea & 63) >> 3) + 2 * (ea & 7);
    const uint32_t ob = (eb >> 6) * kBoxBytes + sw128_off(row, (eb & 63) >> 3) + 2 * (eb & 7);
    uint16_t* pa = reinterpret_cast<uint16_t*>(tile + oa);
    uint16_t* pb = reinterpret_cast<uint16_t*>(tile + ob);
    const float x = __uint_as_float((uint32_t)*pa << 16), y = __uint_as_float((uint32_t)*pb << 16);
    *pa = __bfloat16_as_ushort(__float2bfloat16_rn(fmaf(x, c.x, -(y * c.y))));
    *pb = __bfloat16_as_ushort(__float2bfloat16_rn(fmaf(y, c.x, x * c.y)));
  }
}

// kMode (PrefillMode) is a template parameter so that the whole prefill
// carries neither the query offset nor a per-load layout branch.
template <int kMode>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const PrefillArgs a, const __grid_constant__ CUtensorMap q_map,
                   const __grid_constant__ CUtensorMap k_map, const __grid_constant__ CUtensorMap v_map,
                   const __grid_constant__ CUtensorMap o_map) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // the 128-byte-swizzled tiles need 1024-byte alignment and the layout has
  // no room to realign: leave (uniformly, before any barrier) if it is off
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0) record_error(kErrPrefill + 15);
    return;
  }
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = a.n_q_tiles * a.n_head_pairs * a.Hkv * a.B;

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      for (int s = 0; s < 2; ++s) {
        mbar_init(&sm.q_full[b][s], 1);
        mbar_init(&sm.l_full[b][s], BM);
      }
      mbar_init(&sm.q_ready[b], BM);
      mbar_init(&sm.q_free[b], 1);
    }
    for (int i = 0; i < kKvStages; ++i) {
      mbar_init(&sm.kv_full[i], 1);
      mbar_init(&sm.kv_empty[i], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.s_full[s], 1);
      mbar_init(&sm.p_full[s], BM);
      mbar_init(&sm.o_done[s], 1);
      mbar_init(&sm.o_free[s], BM);
      mbar_init(&sm.o_staged[s], BM);
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

  if (warp >= 12) {
    regs_decrease<kRegsOther>();
    if (warp == 13 && lane == 0) {
      // ========================================================== K / V producer
      // Every key tile j of every work tile, in the order the MMAs consume
      // them: K(j), V(j), into a three-stage ring.
      prefetch_tensormap(&k_map);
      prefetch_tensormap(&v_map);
      int idx = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
        const Tile T = decode_tile<kMode>(a, t);
        for (int j = 0; j < T.n_kv && ok; ++j) {
          const int key0 = (T.kt_lo + j) * BN;
          for (int v = 0; v < 2; ++v, ++idx) {
            const int st = idx % kKvStages;
            if (idx >= kKvStages && !mbar_wait(&sm.kv_empty[st], (idx / kKvStages - 1) & 1, abort_flag)) {
              ok = false;
              break;
            }
            const CUtensorMap* map = v ? &v_map : &k_map;
            uint8_t* dst = sm.kv[st];
            mbar_arrive_expect_tx(&sm.kv_full[st], kTileBytes);
            if constexpr (kMode == kChunkCache) {  // KV cache [B * Hkv, C, D]
              tma_load_3d(dst, map, &sm.kv_full[st], 0, key0, T.b * a.Hkv + T.kvh);
              tma_load_3d(dst + kBoxBytes, map, &sm.kv_full[st], 64, key0, T.b * a.Hkv + T.kvh);
            } else {
              tma_load_4d(dst, map, &sm.kv_full[st], 0, T.kvh, key0, T.b);
              tma_load_4d(dst + kBoxBytes, map, &sm.kv_full[st], 64, T.kvh, key0, T.b);
            }
          }
        }
      }
      if (!ok) {
        fail(abort_flag, kErrPrefill + 1);
        // let every copy this thread started land before the CTA exits
        for (int g = idx > kKvStages ? idx - kKvStages : 0; g < idx; ++g)
          mbar_wait(&sm.kv_full[g % kKvStages], (g / kKvStages) & 1, nullptr, 200000000ull);
      }
    } else if (warp == 15 && lane == 0) {
      // ========================================================== Q producer
      // Q of tile it goes to buffer it & 1 once the output of tile it - 2
      // (the buffer's previous tile), staged there by the epilogue, has been
      // read by its TMA store.
      prefetch_tensormap(&q_map);
      int it = 0, last_it = -1;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++it) {
        const Tile N = decode_tile<kMode>(a, t);
        const int b = it & 1;
        if (it >= 2 && !mbar_wait(&sm.q_free[b], ((it - 2) >> 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        for (int s = 0; s < 2; ++s) {
          const int h = s ? N.h1 : N.h0;
          mbar_arrive_expect_tx(&sm.q_full[b][s], kTileBytes);
          tma_load_4d(sm.q[b][s], &q_map, &sm.q_full[b][s], 0, h, N.r0, N.b);
          tma_load_4d(sm.q[b][s] + kBoxBytes, &q_map, &sm.q_full[b][s], 64, h, N.r0, N.b);
        }
        if (ok) last_it = it;
      }
      if (!ok) {
        fail(abort_flag, kErrPrefill + 2);
        for (int i = last_it > 0 ? last_it - 1 : 0; i <= last_it; ++i)
          for (int s = 0; s < 2; ++s) mbar_wait(&sm.q_full[i & 1][s], (i >> 1) & 1, nullptr, 200000000ull);
      }
    } else if (warp == 12 && lane == 0) {
      // ========================================================== MMA issuer
      // Per key tile j and slot s: [O_s (+)= P_s(j) V(j); S_s = Q_s K(j+1)^T],
      // where after a tile's last key tile K(j+1) is the next tile's first
      // key tile and Q_s the next tile's buffer.  Ring index of K(j) in a tile
      // is base + 2j, of V(j) base + 2j + 1.  Descriptors advance by adding
      // (byte offset >> 4) to the start-address field in their low word.
      constexpr uint32_t idesc_qk = idesc_bf16_f32(BM, BN, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(BM, 128, false, true);
      // the buffers are contiguous, so a buffer's descriptor is the first
      // one's plus its byte offset >> 4 (no carry: shared memory < 256 KB)
      const uint64_t qd = sw128_desc(smem_u32(sm.q[0][0]), 16, 1024);
      const uint64_t kd = sw128_desc(smem_u32(sm.kv[0]), 16, 1024);
      const uint64_t vd = sw128_desc(smem_u32(sm.kv[0]), kBoxBytes, 1024);
      const uint32_t qlo = (uint32_t)qd, qhi = (uint32_t)(qd >> 32);
      const uint32_t klo = (uint32_t)kd, khi = (uint32_t)(kd >> 32);
      const uint32_t vlo = (uint32_t)vd, vhi = (uint32_t)(vd >> 32);
      auto wait_kv = [&](int idx) -> bool {
        return mbar_wait(&sm.kv_full[idx % kKvStages], (idx / kKvStages) & 1, abort_flag);
      };
      auto issue_qk = [&](int b, int s, int kidx) {
        const uint32_t a0 = qlo + (uint32_t)(((b * 2 + s) * kTileBytes) >> 4);
        const uint32_t b0 = klo + (uint32_t)(((kidx % kKvStages) * kTileBytes) >> 4), d = tmem + s * 128;
#pragma unroll 2
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (uint32_t)((((kk >> 2) * kBoxBytes) + (kk & 3) * 32) >> 4);
          umma_ss_lh(d, a0 + off, qhi, b0 + off, khi, idesc_qk, kk > 0);
        }
      };
      auto issue_pv = [&](int s, int vidx, bool acc) {
        const uint32_t b0 = vlo + (uint32_t)(((vidx % kKvStages) * kTileBytes) >> 4);
        const uint32_t d = tmem + 256 + s * 128, pa = tmem + s * 128;
#pragma unroll 2
        for (int kk = 0; kk < 8; ++kk)
          umma_ts_lh(d, pa + kk * 8, b0 + (uint32_t)((kk * 2048) >> 4), vhi, idesc_pv, (acc || kk > 0) ? 1u : 0u);
      };
      bool ok = true;
      int it = 0, g = 0, base = 0;
      if ((int)blockIdx.x < n_tiles) {
        const Tile T0 = decode_tile<kMode>(a, blockIdx.x);
        ok = mbar_wait(&sm.q_ready[0], 0, abort_flag) && wait_kv(0);
        if (ok) {
          tc_fence_after();
          for (int s = 0; s < 2; ++s) {
            issue_qk(0, s, 0);
            umma_commit(&sm.s_full[s]);
          }
          umma_commit(&sm.kv_empty[0]);
        } else {
          fail(abort_flag, kErrPrefill + 3);
        }
      }
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++it) {
        const int n = decode_tile<kMode>(a, t).n_kv;
        const bool has_next = t + (int)gridDim.x < n_tiles;
        const int b = it & 1, nb = b ^ 1;
        for (int j = 0; j < n && ok; ++j) {
          const bool last = j == n - 1;
          const int vidx = base + 2 * j + 1, kidx = base + 2 * j + 2;
          for (int s = 0; s < 2 && ok; ++s) {
            ok = mbar_wait(&sm.p_full[s], (g + j) & 1, abort_flag) &&
                 (j > 0 || it == 0 || mbar_wait(&sm.o_free[s], (it - 1) & 1, abort_flag)) &&
                 (s == 1 || wait_kv(vidx));
            if (!ok) {
              fail(abort_flag, kErrPrefill + 4);
              break;
            }
            tc_fence_after();
            issue_pv(s, vidx, j > 0);
            if (s == 1) umma_commit(&sm.kv_empty[vidx % kKvStages]);
            if (last) umma_commit(&sm.o_done[s]);
            if (!last || has_next) {
              if (s == 0) {
                ok = (!last || mbar_wait(&sm.q_ready[nb], ((it + 1) >> 1) & 1, abort_flag)) && wait_kv(kidx);
                if (!ok) {
                  fail(abort_flag, kErrPrefill + 5);
                  break;
                }
                tc_fence_after();
              }
              issue_qk(last ? nb : b, s, kidx);
              umma_commit(&sm.s_full[s]);
              if (s == 1) umma_commit(&sm.kv_empty[kidx % kKvStages]);
            }
          }
        }
        g += n;
        base += 2 * n;
      }
      // all MMAs issued by this thread complete before the CTA moves on
      umma_commit(&sm.drain);
      mbar_wait(&sm.drain, 0, nullptr, 200000000ull);
    }
  } else if (warp < 8) {
    // ============================================================ softmax
    regs_increase<kRegsSoftmax>();
    const int s = warp >> 2;
    const int row = threadIdx.x & (BM - 1);
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t s_addr = tmem + lane_base + s * 128;
    const uint32_t o_addr = tmem + lane_base + 256 + s * 128;
    const float c = a.scale_log2;
    int it = 0, g = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++it) {
      const Tile T = decode_tile<kMode>(a, t);
      const int i = T.i0 + row;  // key-space position of this row
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < T.n_kv; ++j, ++g) {
        const int key0 = (T.kt_lo + j) * BN;
        if (!warp_wait(&sm.s_full[s], g & 1, abort_flag)) {
          fail(abort_flag, kErrPrefill + 7);
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t v[128];
        tmem_ld32(s_addr + 0, *reinterpret_cast<uint32_t(*)[32]>(v + 0));
        tmem_ld32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
        tmem_ld32(s_addr + 64, *reinterpret_cast<uint32_t(*)[32]>(v + 64));
        tmem_ld32(s_addr + 96, *reinterpret_cast<uint32_t(*)[32]>(v + 96));
        tmem_wait_ld();
        // which mask bounds cut this key tile (uniform over the tile):
        // hi -- some key lies after some row (the diagonal tile);
        // lo -- some key lies at or before row - W (the band's first tile).
        // On a cut tile each 32-column chunk is, for the warp's 32 rows,
        // either wholly masked (skipped: P = 0), wholly visible, or compared
        // column by column.
        const bool cut_hi = key0 + BN - 1 > T.i0;
        const bool cut_lo = a.window > 0 && key0 < T.i0 + BM - a.window;
        uint32_t masked = 0;  // bit q: chunk q masked for every row of the warp
        if (cut_hi || cut_lo) {
          // this row's visible columns are lo .. hi
          const int hi = cut_hi ? i - key0 : BN - 1;
          const int lo = cut_lo ? i - a.window + 1 - key0 : 0;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint32_t keep = chunk_keep(lo - 32 * q, hi - 32 * q);  // bit k: column 32 q + k visible
            if (__all_sync(0xffffffffu, keep == 0u)) {
              masked |= 1u << q;
            } else if (!__all_sync(0xffffffffu, keep == 0xffffffffu)) {
#pragma unroll
              for (int k = 0; k < 32; ++k)
                v[32 * q + k] = ((keep >> k) & 1u) ? v[32 * q + k] : __float_as_uint(-INFINITY);
            }
          }
        }
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (!((masked >> q) & 1u)) {
#pragma unroll
            for (int e = 32 * q; e < 32 * q + 32; e += 2)
              mx[(e >> 1) & 3] = fmax3(mx[(e >> 1) & 3], __uint_as_float(v[e]), __uint_as_float(v[e + 1]));
          }
        }
        const float mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * c;
        const float m_use = (mt - m > kRescaleThreshold) ? mt : m;  // m = -inf: always take mt
        const float m_safe = m_use == -INFINITY ? 0.f : m_use;
        // a row that has seen no visible key yet has O = 0 and l = 0: it
        // needs no rescale (alpha 1 keeps the band-edge tile's emptiest row
        // from sending its whole warp through the O rescale)
        const float alpha = m == -INFINITY ? 1.f : fast_exp2(m - m_safe);
        // P = 2^(c S - m), two columns per packed FMA; masked columns give 0
        const uint64_t cc = f2_pack(c, c), mm = f2_pack(-m_safe, -m_safe);
        uint64_t sum2[4] = {0ull, 0ull, 0ull, 0ull};
        uint32_t pk[64];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if ((masked >> q) & 1u) {
#pragma unroll
            for (int e = 32 * q; e < 32 * q + 32; e += 2) pk[e >> 1] = 0u;
          } else {
#pragma unroll
            for (int e = 32 * q; e < 32 * q + 32; e += 2) {
              const uint64_t y = f2_fma(f2_pack(__uint_as_float(v[e]), __uint_as_float(v[e + 1])), cc, mm);
              float y0, y1;
              f2_unpack(y, y0, y1);
              const float p0 = fast_exp2(y0), p1 = fast_exp2(y1);
              sum2[(e >> 1) & 3] = f2_add(sum2[(e >> 1) & 3], f2_pack(p0, p1));
              pk[e >> 1] = pack_bf16x2(p0, p1);
            }
          }
        }
        // P over the S columns it came from (S is in registers already)
        tmem_st32(s_addr + 0, *reinterpret_cast<const uint32_t(*)[32]>(pk + 0));
        tmem_st32(s_addr + 32, *reinterpret_cast<const uint32_t(*)[32]>(pk + 32));
        // O_s holds key tiles 0..j-1 (their P.V completed before S(j) did):
        // bring it to the new max before P(j).V adds to it
        if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
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
        mbar_arrive(&sm.p_full[s]);
        float s0, s1;
        f2_unpack(f2_add(f2_add(sum2[0], sum2[1]), f2_add(sum2[2], sum2[3])), s0, s1);
        l = l * alpha + (s0 + s1);
        m = m_use;
      }
      if (!ok) break;
      // double-buffered by tile parity: the epilogue of tile it - 2 read this
      // slot before tile it's first P.V could start
      sm.lsum[it & 1][s][row] = l;
      mbar_arrive(&sm.l_full[it & 1][s]);
    }
  } else {
    // ============================================================ Q rotation + epilogue
    regs_decrease<kRegsCorrection>();
    const int row = threadIdx.x & (BM - 1);
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const int half = a.rotary_dim / 2;
    const bool vec = (half & 7) == 0;
    // RoPE of the Q tiles of work tile tq (iteration itq) in buffer itq & 1,
    // both head slots, this thread's row (rows at or beyond S stay as
    // loaded: zero)
    auto rotate = [&](int tq, int itq) -> bool {
      const Tile N = decode_tile<kMode>(a, tq);
      const int b = itq & 1;
      const int r = N.r0 + row;
      const bool rot = half > 0 && r < a.S;
      const float4* tgroup = reinterpret_cast<const float4*>(a.table) +
                             ((((size_t)(r >> 5) * rope_table_couples(half)) << 5) + (r & 31));
      // the next chunk's table slices (eight pairs) are in flight while the
      // current chunk is applied; slices past the last chunk repeat it
      const int n_chunks = half / 8;
      float4 ta[4], tb[4];
      auto load1 = [&](float4 (&t)[4], int c0) {
#pragma unroll
        for (int w = 0; w < 4; ++w) t[w] = __ldg(tgroup + (size_t)(4 * min(c0, n_chunks - 1) + w) * 32);
      };
      if (rot && vec) load1(ta, 0);
      if (!warp_wait(&sm.q_full[b][0], (itq >> 1) & 1, abort_flag) ||
          !warp_wait(&sm.q_full[b][1], (itq >> 1) & 1, abort_flag))
        return false;
      if (rot) {
        if (vec) {
          for (int c0 = 0; c0 < n_chunks; c0 += 2) {
            load1(tb, c0 + 1);
            rotate_q_chunk(sm.q[b][0], row, c0, half, ta);
            rotate_q_chunk(sm.q[b][1], row, c0, half, ta);
            if (c0 + 1 >= n_chunks) break;
            load1(ta, c0 + 2);
            rotate_q_chunk(sm.q[b][0], row, c0 + 1, half, tb);
            rotate_q_chunk(sm.q[b][1], row, c0 + 1, half, tb);
          }
        } else {
          rotate_q_row_scalar(sm.q[b][0], row, r, half, a.table);
          rotate_q_row_scalar(sm.q[b][1], row, r, half, a.table);
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&sm.q_ready[b]);
      return true;
    };
    int it = 0;
    bool ok = true;
    if ((int)blockIdx.x < n_tiles && !rotate(blockIdx.x, 0)) {
      fail(abort_flag, kErrPrefill + 6);
      ok = false;
    }
    for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++it) {
      const Tile T = decode_tile<kMode>(a, t);
      const int r = T.r0 + row;  // query row
      // gate logits of this row for both head slots, fetched early
      float glog0 = 0.f, glog1 = 0.f;
      if (a.gate && r < a.S) {
        glog0 = __ldg(a.gate + ((size_t)T.b * a.S + r) * a.Hq + T.h0);
        glog1 = __ldg(a.gate + ((size_t)T.b * a.S + r) * a.Hq + T.h1);
      }
      if (t + (int)gridDim.x < n_tiles && !rotate(t + gridDim.x, it + 1)) {
        fail(abort_flag, kErrPrefill + 8);
        break;
      }
      // ---- epilogue: out = O / l * sigmoid(gate), bf16, staged in this
      // tile's Q buffers (their last QK^T completed before O did) and
      // written by TMA stores; the Q producer refills the buffers once the
      // stores have read them
      const int b = it & 1;
      for (int s = 0; s < 2 && ok; ++s) {
        if (!warp_wait(&sm.o_done[s], it & 1, abort_flag) ||
            !warp_wait(&sm.l_full[b][s], (it >> 1) & 1, abort_flag)) {
          fail(abort_flag, kErrPrefill + 11);
          ok = false;
          break;
        }
        tc_fence_after();
        const float l = sm.lsum[b][s][row];
        const float gt = a.gate ? 1.f / (1.f + __expf(-(s ? glog1 : glog0))) : 1.f;
        const float f = gt / l;
        uint8_t* stage = sm.q[b][s];
        const uint32_t oaddr = tmem + lane_base + 256 + s * 128;
#pragma unroll 1
        for (int q4 = 0; q4 < 4; ++q4) {
          uint32_t v[32];
          tmem_ld32(oaddr + q4 * 32, v);
          tmem_wait_ld();
          if (q4 == 3) {
            // O_s is in registers: the next tile's first P.V may overwrite it
            tc_fence_before();
            mbar_arrive(&sm.o_free[s]);
          }
          uint8_t* box = stage + (q4 >> 1) * kBoxBytes;
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            uint4 u;
            u.x = pack_bf16x2(__uint_as_float(v[8 * c4 + 0]) * f, __uint_as_float(v[8 * c4 + 1]) * f);
            u.y = pack_bf16x2(__uint_as_float(v[8 * c4 + 2]) * f, __uint_as_float(v[8 * c4 + 3]) * f);
            u.z = pack_bf16x2(__uint_as_float(v[8 * c4 + 4]) * f, __uint_as_float(v[8 * c4 + 5]) * f);
            u.w = pack_bf16x2(__uint_as_float(v[8 * c4 + 6]) * f, __uint_as_float(v[8 * c4 + 7]) * f);
            *reinterpret_cast<uint4*>(box + sw128_off(row, (q4 & 1) * 4 + c4)) = u;
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(&sm.o_staged[s]);
        if (threadIdx.x == 256) {
          // one thread stores the tile (rows at or beyond S are clipped by
          // the tensor map); a time-out only records the error and sets the
          // abort flag, so that the warp's lanes stay on one path
          if (!mbar_wait(&sm.o_staged[s], it & 1, abort_flag)) {
            fail(abort_flag, kErrPrefill + 12);
          } else if (s == 0 || T.store1) {
            const int h = s ? T.h1 : T.h0;
            tma_store_4d(&o_map, stage, 0, h, T.r0, T.b);
            tma_store_4d(&o_map, stage + kBoxBytes, 64, h, T.r0, T.b);
            bulk_commit_group();
          }
        }
      }
      if (threadIdx.x == 256) {
        bulk_wait_group_read0();
        mbar_arrive(&sm.q_free[b]);
      }
    }
    // the output stores complete before the CTA exits
    if (threadIdx.x == 256) bulk_wait_group0();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int kMode>
cudaError_t launch_prefill_t(const PrefillArgs& a, const CUtensorMap& q_map, const CUtensorMap& k_map,
                             const CUtensorMap& v_map, const CUtensorMap& o_map, cudaStream_t stream) {
  const long long n_tiles = (long long)a.n_q_tiles * a.n_head_pairs * a.Hkv * a.B;
  if (n_tiles == 0) return cudaSuccess;
  if (n_tiles > 0x7FFFFFFFll) return cudaErrorInvalidConfiguration;
  const size_t smem = sizeof(Smem);
  static DeviceOnce setup;
  int n_sm = 0;
  cudaError_t e = device_once(setup, [&](int dev, int* sm_count) -> cudaError_t {
    cudaError_t r =
        cudaFuncSetAttribute(prefill_kernel<kMode>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (r != cudaSuccess) return r;
    // setmaxnreg redistributes the registers the CTA was launched with: the
    // kernel must be launched with exactly kRegsLaunch per thread
    cudaFuncAttributes fa;
    r = cudaFuncGetAttributes(&fa, prefill_kernel<kMode>);
    if (r != cudaSuccess) return r;
    if (fa.numRegs != (int)kRegsLaunch) return cudaErrorInvalidConfiguration;
    return cudaDeviceGetAttribute(sm_count, cudaDevAttrMultiProcessorCount, dev);
  }, &n_sm);
  if (e != cudaSuccess) return e;
  const int grid = (int)(n_tiles < n_sm ? n_tiles : n_sm);
  return launch_kernel(false, prefill_kernel<kMode>, dim3(grid), dim3(kThreads), smem, stream, a, q_map, k_map,
                       v_map, o_map);
}

}  // namespace prefill_detail

cudaError_t launch_prefill(const PrefillArgs& a, const CUtensorMap& q_map, const CUtensorMap& k_map,
                            const CUtensorMap& v_map, const CUtensorMap& o_map, cudaStream_t stream) {
  using namespace prefill_detail;
  if (a.kv_cache_layout) return launch_prefill_t<kChunkCache>(a, q_map, k_map, v_map, o_map, stream);
  if (a.q_off) return launch_prefill_t<kChunkSeq>(a, q_map, k_map, v_map, o_map, stream);
  return launch_prefill_t<kWhole>(a, q_map, k_map, v_map, o_map, stream);
}

}  // namespace swa
