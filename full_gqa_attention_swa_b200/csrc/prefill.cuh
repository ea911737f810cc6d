// Prefill attention on sm_100a: RoPE'd Q, banded causal mask, GQA, online
// softmax, P.V and the per-head sigmoid gate, with tcgen05 tensor-core MMAs
// accumulating in tensor memory, TMA loads into shared memory and a TMA
// store of the output.
//
// Follows the "Step-3.7-Flash-oQ3e" explainer: section 2.2 (sliding-window
// causal mask of W keys on sliding layers, plain causal mask on full layers)
// and section 2.3 (per-layer rope theta, partial rotary, head-wise sigmoid
// gate); the "Step-3.7-Flash" spec card's GQA groups; the "Muse-Glimmer-30B-
// 6bit" explainer's theta = 0 (no rotation) on full layers.
//
// Work unit ("tile"): 128 query rows x two q-heads of the same kv-head, so
// every K/V tile in shared memory feeds two 128x128 score tiles.  Query row r
// sits at key-space position i = q_off + r (q_off > 0 when a chunk of queries
// continues a sequence whose earlier keys are in the K/V source).  A tile
// loops over the key tiles of its band [i0 - W + 1, i0 + 127]; key tiles
// wholly outside the band are never loaded, and the mask is evaluated only
// on tiles the band edge or the diagonal cuts.  The grid is persistent (one
// CTA per SM); a CTA walks tiles blockIdx.x, +gridDim.x, ... in an order
// that puts the longest (latest-row) tiles first.  Loads, rotation and the
// output store of neighbouring tiles overlap with the tensor-core work.
//
// Warp roles (16 warps, registers rebalanced with setmaxnreg):
//   warps 0-3   head slot 0: Q rotation, softmax (thread = query row)
//   warps 4-7   head slot 1: same
//   warps 8-11  O rescaling ("correction") and the epilogue (O/l * gate ->
//               bf16 -> the slot's P buffer in shared memory)
//   warp 12     tcgen05.mma issuer (one thread)
//   warp 13     TMA producer (one thread)
//   warp 14     TMA store of the output tiles (one thread)
//   warp 15     folds K / V arrivals into the issuer's barriers (one thread)
// Tensor memory (512 columns): S0 [0,128) S1 [128,256) O0 [256,384)
// O1 [384,512).  P (bf16) goes to a shared-memory buffer per head slot.
//
// Per key tile j and head slot s:
//   MMA:     S_s = Q_s K_j^T            -> s_full (both slots)
//   softmax: read S_s                   -> s_free (both slots: S(j+1) may start)
//            m, alpha                   -> alpha_full[s]
//            P_s = 2^(S_s - m) -> smem  -> pv_ready
//   correct: wait PV_s(j-1), O_s *= alpha (skipped when alpha == 1 for the
//            whole warp)                -> pv_ready
//   MMA:     O_s += P_s V_j             -> pv_done (both slots; frees the P buffers)
// The MMA thread waits on one barrier per hand-off (s_free, pv_ready) rather
// than one per slot and producer: each wait is a shared-memory round trip that
// queues behind the softmax warps' SFU traffic on the same sub-partition.  A
// helper thread folds the K / V tile arrivals into those two barriers.
// The exponentials run on the SFU (a polynomial path on the FMA pipe exists,
// see poly_column_pair).
// The max used for the exponentials only moves when the new row max exceeds
// it by more than 8 (log2 units), so most tiles need no O rescale; exp2 of a
// score then stays below 2^8, and the final normalisation by the row sum
// computed with the same max is exact.
#pragma once
#include "swa_internal.cuh"

namespace swa {

namespace prefill_detail {

constexpr int BM = 128;                         // query rows per tile
constexpr int BN = 128;                         // keys per key tile
constexpr int NK = 2;                           // K tile ring
constexpr int NV = 1;                           // V tile ring
constexpr int kThreads = 512;
constexpr uint32_t kBoxBytes = 128 * 128;       // 128 rows x 64 bf16
constexpr uint32_t kTileBytes = 2 * kBoxBytes;  // 128 rows x 128 bf16
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;       // log2 units

// setmaxnreg split of the 128 x 512 registers the CTA is launched with
constexpr uint32_t kRegsLaunch = 128;
constexpr uint32_t kRegsSoftmax = 176;
constexpr uint32_t kRegsCorrection = 104;
constexpr uint32_t kRegsOther = 56;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsCorrection + 128 * kRegsOther <= kRegsLaunch * kThreads,
              "register split exceeds the launch allocation");

// 231,712 bytes: within the 232,448-byte opt-in limit only because the
// dynamic shared memory window starts 1024-byte aligned (checked at entry).
struct PrefillSmem {
  uint8_t q[2][kTileBytes];    // Q of each head slot (rotated in place)
  uint8_t p[2][kTileBytes];    // P (bf16) of each slot; also stages its output tile
  uint8_t k[NK][kTileBytes];
  uint8_t v[NV][kTileBytes];
  float alpha[2][BM];
  float lsum[2][BM];
  uint64_t q_full[2], q_empty[2];
  uint64_t q_ready;  // both slots' Q rotated (256 arrivals)
  uint64_t k_full[NK], k_empty[NK], v_full[NV], v_empty[NV];
  uint64_t alpha_full[2], alpha_empty[2];
  uint64_t s_full;    // S of both slots complete
  uint64_t pv_done;   // P.V of both slots complete (frees both P buffers)
  uint64_t s_free;    // both slots have read S, and the next K tile has landed (256 + 1 arrivals)
  uint64_t pv_ready;  // both slots' P written and O rescaled, and the V tile has landed (512 + 1)
  uint64_t l_full[2], l_empty[2];
  uint64_t ost_full[2];  // output tile staged in p[s]
  uint64_t pfree[2];     // the store of that tile has read p[s]
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

// Column pairs (of every 8) whose exponentials run on the FMA pipe
// (exp2_poly2) instead of the SFU.  Zero: the step is bound by the tensor
// pipe and the MMA thread's hand-offs, not by the SFU, and the polynomial's
// extra issue slots on the MMA thread's sub-partition slow it (by 5-8% at 3 of
// 8 pairs).
constexpr int kPolyPairsPer8 = 0;
__host__ __device__ constexpr bool poly_column_pair(int pair) { return (pair & 7) < kPolyPairsPer8; }

__device__ __forceinline__ uint32_t sw128_off(int row, int chunk) {
  return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
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

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// Rotate query row `row` (position i) of the Q tiles in shared memory (two
// 64-dim boxes, 128-byte swizzle): pairs (k, k + r/2) for k < r/2.  Vector
// form for 16 | r.  Both head slots' tiles hold the same query rows, so the
// slots split a row's 8-pair chunks between them (slot s takes chunks
// c0 = s, s+2, s+4, s+6) and each rotates its chunks in both tiles: every
// table slice crosses from L2 once per work tile.  tb holds the thread's
// 16-byte slices (two pairs each), loaded before the tiles' arrival is
// awaited; the warp's 32 rows load each slice index from 512 contiguous
// bytes.
__device__ __forceinline__ void rope_table_load(float4 (&tb)[16], const float4* __restrict__ tgroup, int half,
                                                int slot) {
  // slices past half/2 repeat the last one: unconditional loads stay in registers
  const int last = half / 2 - 1;
#pragma unroll
  for (int ci = 0; ci < 4; ++ci)
#pragma unroll
    for (int w = 0; w < 4; ++w) tb[4 * ci + w] = __ldg(tgroup + (size_t)min((2 * ci + slot) * 4 + w, last) * 32);
}

// Rotates dims 8 c0 .. 8 c0 + 7 with their partners 8 c0 + half .. of one row;
// t4[w] holds (cos, sin) of pairs 8 c0 + 2w and 8 c0 + 2w + 1.
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
    // the partner's product rounded, then one fma: the RoPE kernels' form,
    // so a rotated q equals swa_rope_qk's bit for bit
    a32[w] = pack_bf16x2(fmaf(x0, t.x, -(y0 * t.y)), fmaf(x1, t.z, -(y1 * t.w)));
    b32[w] = pack_bf16x2(fmaf(y0, t.x, x0 * t.y), fmaf(y1, t.z, x1 * t.w));
  }
  *pa = A;
  *pb = Bv;
}

__device__ __forceinline__ void rotate_q_rows_vec(uint8_t* q0, uint8_t* q1, int row, int half, int slot,
                                                  const float4 (&tb)[16]) {
#pragma unroll
  for (int ci = 0; ci < 4; ++ci) {
    const int c0 = 2 * ci + slot;
    if (c0 * 8 < half) {
      rotate_q_chunk(q0, row, c0, half, tb + 4 * ci);
      rotate_q_chunk(q1, row, c0, half, tb + 4 * ci);
    }
  }
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
  PrefillSmem& sm = *reinterpret_cast<PrefillSmem*>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = a.n_q_tiles * a.n_head_pairs * a.Hkv * a.B;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.q_full[s], 1);
      mbar_init(&sm.q_empty[s], 1);
      mbar_init(&sm.alpha_full[s], BM);
      mbar_init(&sm.alpha_empty[s], BM);
      mbar_init(&sm.l_full[s], BM);
      mbar_init(&sm.l_empty[s], BM);
      mbar_init(&sm.ost_full[s], BM);
      mbar_init(&sm.pfree[s], 1);
    }
    for (int i = 0; i < NK; ++i) {
      mbar_init(&sm.k_full[i], 1);
      mbar_init(&sm.k_empty[i], 1);
    }
    for (int i = 0; i < NV; ++i) {
      mbar_init(&sm.v_full[i], 1);
      mbar_init(&sm.v_empty[i], 1);
    }
    mbar_init(&sm.q_ready, 2 * BM);
    mbar_init(&sm.s_full, 1);
    mbar_init(&sm.pv_done, 1);
    mbar_init(&sm.s_free, 2 * BM + 1);
    mbar_init(&sm.pv_ready, 4 * BM + 1);
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
      // ========================================================== producer
      // Per work tile: K(0), then [K(j+1), V(j)] per key tile (K runs one
      // ahead, its 2-deep ring frees early; V's single buffer frees when both
      // slots' P.V of the previous key tile complete).  The next tile's Q is
      // loaded as soon as this tile's last QK^T has read Q.  No L2 prefetches
      // (of the next V, or of a later tile's Q and cos/sin rows): with them
      // the loads queued behind land later and the step is about 2 % slower.
      prefetch_tensormap(&q_map);
      prefetch_tensormap(&k_map);
      prefetch_tensormap(&v_map);
      int it = 0, kc = 0, vc = 0;           // tile counter, K / V loads issued
      int k_end = 0, v_end = 0;             // loads issued (for the abort drain)
      int q_last[2] = {-1, -1};
      bool ok = true;
      auto load_q = [&](int t_q, int it_q) -> bool {
        const Tile N = decode_tile<kMode>(a, t_q);
        for (int s = 0; s < 2; ++s) {
          if (it_q > 0 && !mbar_wait(&sm.q_empty[s], (it_q - 1) & 1, abort_flag)) return false;
          mbar_arrive_expect_tx(&sm.q_full[s], kTileBytes);
          const int h = s ? N.h1 : N.h0;
          tma_load_4d(sm.q[s], &q_map, &sm.q_full[s], 0, h, N.r0, N.b);
          tma_load_4d(sm.q[s] + kBoxBytes, &q_map, &sm.q_full[s], 64, h, N.r0, N.b);
          q_last[s] = it_q;
        }
        return true;
      };
      auto load_kv = [&](bool is_v, const Tile& T, int j) -> bool {
        const int idx = is_v ? vc++ : kc++;
        const int nb = is_v ? NV : NK;
        const int buf = idx % nb, use = idx / nb;
        uint64_t* full = is_v ? &sm.v_full[buf] : &sm.k_full[buf];
        uint64_t* empty = is_v ? &sm.v_empty[buf] : &sm.k_empty[buf];
        if (use > 0 && !mbar_wait(empty, (use - 1) & 1, abort_flag)) return false;
        uint8_t* dst = is_v ? sm.v[buf] : sm.k[buf];
        const CUtensorMap* map = is_v ? &v_map : &k_map;
        const int key0 = (T.kt_lo + j) * BN;
        mbar_arrive_expect_tx(full, kTileBytes);
        if constexpr (kMode == kChunkCache) {  // KV cache [B * Hkv, C, D]
          tma_load_3d(dst, map, full, 0, key0, T.b * a.Hkv + T.kvh);
          tma_load_3d(dst + kBoxBytes, map, full, 64, key0, T.b * a.Hkv + T.kvh);
        } else {
          tma_load_4d(dst, map, full, 0, T.kvh, key0, T.b);
          tma_load_4d(dst + kBoxBytes, map, full, 64, T.kvh, key0, T.b);
        }
        if (is_v)
          v_end = idx + 1;
        else
          k_end = idx + 1;
        return true;
      };
      if (blockIdx.x < (unsigned)n_tiles && !load_q(blockIdx.x, 0)) ok = false;
      for (int t = blockIdx.x; t < n_tiles && ok && !*abort_flag; t += gridDim.x, ++it) {
        const Tile T = decode_tile<kMode>(a, t);
        const bool has_next = t + (int)gridDim.x < n_tiles;
        for (int j = -1; j < T.n_kv && ok; ++j) {
          if (j + 1 < T.n_kv) ok = load_kv(false, T, j + 1);
          if (ok && j >= 0) {
            // the next tile's Q waits for this tile's last QK^T: issue it
            // before the last V (which waits for the previous P.V), or after
            // the only V of a one-key-tile tile
            const bool last = j == T.n_kv - 1;
            if (last && has_next && T.n_kv >= 2) ok = load_q(t + gridDim.x, it + 1);
            if (ok) ok = load_kv(true, T, j);
            if (ok && last && has_next && T.n_kv == 1) ok = load_q(t + gridDim.x, it + 1);
          }
        }
        if (!ok) fail(abort_flag, kErrPrefill + 1);
      }
      if (*abort_flag) {
        // let every copy this thread started land before the CTA exits
        for (int s = 0; s < 2; ++s)
          if (q_last[s] >= 0) mbar_wait(&sm.q_full[s], q_last[s] & 1, nullptr, 200000000ull);
        for (int g = k_end > NK ? k_end - NK : 0; g < k_end; ++g)
          mbar_wait(&sm.k_full[g % NK], (g / NK) & 1, nullptr, 200000000ull);
        for (int g = v_end > NV ? v_end - NV : 0; g < v_end; ++g)
          mbar_wait(&sm.v_full[g % NV], (g / NV) & 1, nullptr, 200000000ull);
      }
    } else if (warp == 12 && lane == 0) {
      // ========================================================== MMA issuer
      // In-phase order per key tile: [S_0(j+1), S_1(j+1)] then [O_0 += P_0 V_j,
      // O_1 += P_1 V_j], each pair issued one MMA of each GEMM in turn.  S(j+1)
      // needs only that the softmax has read S(j) (P is in shared memory), so
      // both QK^T of the next key tile overlap the softmax and the P.V of the
      // current one: up to four independent accumulation chains in the pipe,
      // where a lone chain of dependent tcgen05.mma runs at a fraction of its
      // rate.  Descriptors advance by adding (byte offset >> 4) to the
      // start-address field (no carry below 256 KB).
      constexpr uint32_t idesc_qk = idesc_bf16_f32(BM, BN, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(BM, 128, false, true);
      const uint64_t qd0 = sw128_desc(smem_u32(sm.q[0]), 16, 1024), qd1 = sw128_desc(smem_u32(sm.q[1]), 16, 1024);
      const uint64_t pd0 = sw128_desc(smem_u32(sm.p[0]), 16, 1024), pd1 = sw128_desc(smem_u32(sm.p[1]), 16, 1024);
      const uint64_t kdesc0 = sw128_desc(smem_u32(sm.k[0]), 16, 1024);
      const uint64_t vdesc0 = sw128_desc(smem_u32(sm.v[0]), kBoxBytes, 1024);
      int it = 0, G = 0, kc = 0, vc = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++it) {
        const int n_kv = decode_tile<kMode>(a, t).n_kv;
        if (!mbar_wait(&sm.q_ready, it & 1, abort_flag)) {
          fail(abort_flag, kErrPrefill + 3);
          ok = false;
          break;
        }
        for (int j = -1; j < n_kv && ok; ++j) {
          if (j + 1 < n_kv) {
            const int g1 = G + j + 1, ki = kc + j + 1;
            // s_free(g1 - 1) includes the arrival of K(g1); only the very
            // first K tile is awaited here
            ok = g1 == 0 ? mbar_wait(&sm.k_full[0], 0, abort_flag) : mbar_wait(&sm.s_free, (g1 - 1) & 1, abort_flag);
            if (!ok) {
              fail(abort_flag, kErrPrefill + 4);
              break;
            }
            tc_fence_after();
            const uint64_t kd = kdesc0 + (uint64_t)(((ki % NK) * kTileBytes) >> 4);
            // unrolled by 2, descriptors advanced in their low words: fewer
            // instructions between MMAs on the issuer's busy sub-partition (C2
            // -1.7 % and -2.2 %, C3 -2.9 % and -2.1 %; fully unrolled it spills at
            // this warp's 56 registers, by 4 it ran slower)
#pragma unroll 2
            for (int kk = 0; kk < 8; ++kk) {
              const uint64_t off = (uint64_t)((((kk >> 2) * kBoxBytes) + (kk & 3) * 32) >> 4);
              const uint32_t o32 = (uint32_t)off;
              umma_ss_lh(tmem, (uint32_t)qd0 + o32, (uint32_t)(qd0 >> 32), (uint32_t)kd + o32, (uint32_t)(kd >> 32),
                         idesc_qk, kk > 0);
              umma_ss_lh(tmem + 128, (uint32_t)qd1 + o32, (uint32_t)(qd1 >> 32), (uint32_t)kd + o32,
                         (uint32_t)(kd >> 32), idesc_qk, kk > 0);
            }
            umma_commit(&sm.s_full);
            umma_commit(&sm.k_empty[ki % NK]);
            if (j + 2 == n_kv) {
              umma_commit(&sm.q_empty[0]);
              umma_commit(&sm.q_empty[1]);
            }
          }
          if (j >= 0) {
            const int g = G + j, vi = vc + j;
            ok = mbar_wait(&sm.pv_ready, g & 1, abort_flag);  // includes the arrival of V(g)
            if (!ok) {
              fail(abort_flag, kErrPrefill + 5);
              break;
            }
            tc_fence_after();
            const uint64_t vd = vdesc0 + (uint64_t)(((vi % NV) * kTileBytes) >> 4);
#pragma unroll 2
            for (int kk = 0; kk < 8; ++kk) {
              const uint64_t aoff = (uint64_t)((((kk >> 2) * kBoxBytes) + (kk & 3) * 32) >> 4);
              const uint64_t boff = (uint64_t)((kk * 2048) >> 4);
              const uint32_t acc = (j > 0 || kk > 0) ? 1u : 0u;
              umma_ss_lh(tmem + 256, (uint32_t)pd0 + (uint32_t)aoff, (uint32_t)(pd0 >> 32), (uint32_t)vd + (uint32_t)boff,
                         (uint32_t)(vd >> 32), idesc_pv, acc);
              umma_ss_lh(tmem + 384, (uint32_t)pd1 + (uint32_t)aoff, (uint32_t)(pd1 >> 32), (uint32_t)vd + (uint32_t)boff,
                         (uint32_t)(vd >> 32), idesc_pv, acc);
            }
            umma_commit(&sm.pv_done);
            umma_commit(&sm.v_empty[vi % NV]);
          }
        }
        G += n_kv;
        kc += n_kv;
        vc += n_kv;
      }
      // all MMAs issued by this thread complete before the CTA moves on
      umma_commit(&sm.drain);
      mbar_wait(&sm.drain, 0, nullptr, 200000000ull);
    } else if (warp == 15 && lane == 0) {
      // ========================================================== arrivals
      // Folds the landing of each K / V tile into the barrier the MMA thread
      // waits on anyway: s_free(g - 1) counts the arrival of K(g), pv_ready(g)
      // that of V(g), in the issuer's order.  Before arriving for a phase it
      // waits for the previous phase to complete, so an early arrival never
      // counts toward the wrong phase.
      int G = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
        const int n_kv = decode_tile<kMode>(a, t).n_kv;
        for (int j = -1; j < n_kv && ok; ++j) {
          const int g1 = G + j + 1;
          if (j + 1 < n_kv && g1 >= 1) {
            ok = (g1 < 2 || mbar_wait(&sm.s_free, (g1 - 2) & 1, abort_flag)) &&
                 mbar_wait(&sm.k_full[g1 % NK], (g1 / NK) & 1, abort_flag);
            if (ok) mbar_arrive(&sm.s_free);
          }
          if (ok && j >= 0) {
            const int g = G + j;
            ok = (g < 1 || mbar_wait(&sm.pv_ready, (g - 1) & 1, abort_flag)) &&
                 mbar_wait(&sm.v_full[g % NV], (g / NV) & 1, abort_flag);
            if (ok) mbar_arrive(&sm.pv_ready);
          }
        }
        G += n_kv;
      }
      if (!ok) fail(abort_flag, kErrPrefill + 18);
    } else if (warp == 14 && lane == 0) {
      // ========================================================== output store
      // The epilogue stages each slot's output tile in that slot's P buffer;
      // this thread stores it with TMA and frees the buffer once it is read.
      prefetch_tensormap(&o_map);
      int it = 0;
      for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++it) {
        const Tile T = decode_tile<kMode>(a, t);
        bool ok = true;
        for (int s = 0; s < 2; ++s) {
          if (!mbar_wait(&sm.ost_full[s], it & 1, abort_flag)) {
            fail(abort_flag, kErrPrefill + 14);
            ok = false;
            break;
          }
          if (s == 0 || T.store1) {
            const int h = s ? T.h1 : T.h0;
            tma_store_4d(&o_map, sm.p[s], 0, h, T.r0, T.b);
            tma_store_4d(&o_map, sm.p[s] + kBoxBytes, 64, h, T.r0, T.b);
            bulk_commit_group();
          }
          bulk_wait_group_read0();
          mbar_arrive(&sm.pfree[s]);
        }
        if (!ok) break;
      }
      bulk_wait_group0();
    }
  } else if (warp < 8) {
    // ============================================================ softmax
    regs_increase<kRegsSoftmax>();
    const int s = warp >> 2;
    const int row = threadIdx.x & (BM - 1);
    const uint32_t taddr = tmem + ((uint32_t)((warp & 3) * 32) << 16) + s * 128;
    const float c = a.scale_log2;
    int it = 0, G = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++it) {
      const Tile T = decode_tile<kMode>(a, t);
      const int r = T.r0 + row;  // query row
      const int i = T.i0 + row;  // its key-space position
      // ---- RoPE of the Q tiles (rows at or beyond S stay as loaded: zero);
      // the table slices are requested before Q is awaited.  Vector form:
      // this slot's half of each row's chunks in both tiles; scalar form:
      // this slot's own tile.
      {
        const int half = a.rotary_dim / 2;
        const bool rot = a.rotary_dim > 0 && r < a.S;
        const bool vec = (half & 7) == 0;
        const float4* tgroup = reinterpret_cast<const float4*>(a.table) +
                               ((((size_t)(r >> 5) * rope_table_couples(half)) << 5) + (r & 31));
        float4 tb[16];
        if (rot && vec) {
          rope_table_load(tb, tgroup, half, s);
        } else {
#pragma unroll
          for (int k = 0; k < 16; ++k) tb[k] = make_float4(1.f, 0.f, 1.f, 0.f);
        }
        if (!warp_wait(&sm.q_full[0], it & 1, abort_flag) || !warp_wait(&sm.q_full[1], it & 1, abort_flag)) {
          fail(abort_flag, kErrPrefill + 6);
          ok = false;
          break;
        }
        if (rot) {
          if (vec)
            rotate_q_rows_vec(sm.q[0], sm.q[1], row, half, s, tb);
          else
            rotate_q_row_scalar(sm.q[s], row, r, half, a.table);
        }
        fence_proxy_async_smem();
        mbar_arrive(&sm.q_ready);
      }
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < T.n_kv; ++j) {
        const int key0 = (T.kt_lo + j) * BN;
        if (!warp_wait(&sm.s_full, (G + j) & 1, abort_flag)) {
          fail(abort_flag, kErrPrefill + 7);
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t v[128];
        tmem_ld32(taddr + 0, *reinterpret_cast<uint32_t(*)[32]>(v + 0));
        tmem_ld32(taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
        tmem_ld32(taddr + 64, *reinterpret_cast<uint32_t(*)[32]>(v + 64));
        tmem_ld32(taddr + 96, *reinterpret_cast<uint32_t(*)[32]>(v + 96));
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&sm.s_free);  // S_s may be overwritten by the next QK^T
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
          const int hi = cut_hi ? i - key0 : BN;                     // columns > hi are masked
          const int lo = cut_lo ? i - a.window + 1 - key0 : -1;      // columns < lo are masked
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int c0 = 32 * q;
            if (__all_sync(0xffffffffu, hi < c0 || lo > c0 + 31)) {
              masked |= 1u << q;
            } else if (!__all_sync(0xffffffffu, lo <= c0 && hi >= c0 + 31)) {
#pragma unroll
              for (int e = c0; e < c0 + 32; ++e)
                if (e > hi || e < lo) v[e] = __float_as_uint(-INFINITY);
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
        const float alpha = fast_exp2(m - m_safe);
        // the correction has read the previous alpha (the softmax can run a
        // key tile ahead of it now that S(j+1) no longer waits for P(j).V)
        if (G + j > 0 && !warp_wait(&sm.alpha_empty[s], (G + j - 1) & 1, abort_flag)) {
          fail(abort_flag, kErrPrefill + 17);
          ok = false;
          break;
        }
        sm.alpha[s][row] = alpha;
        mbar_arrive(&sm.alpha_full[s]);
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
              float p0, p1;
              if (poly_column_pair(e >> 1)) {
                f2_unpack(exp2_poly2(y), p0, p1);
              } else {
                float y0, y1;
                f2_unpack(y, y0, y1);
                p0 = fast_exp2(y0);
                p1 = fast_exp2(y1);
              }
              sum2[(e >> 1) & 3] = f2_add(sum2[(e >> 1) & 3], f2_pack(p0, p1));
              pk[e >> 1] = pack_bf16x2(p0, p1);
            }
          }
        }
        // p[s] is free once P_s(j-1).V has completed; at a tile's first key
        // tile it holds the previous tile's output until the store has read
        // it.  (S(j) completing implies P(j-2).V completed, since its commit
        // covers every earlier MMA, so these waits are never two phases ahead.)
        if (j > 0 ? !warp_wait(&sm.pv_done, (G + j - 1) & 1, abort_flag)
                  : (it > 0 && !warp_wait(&sm.pfree[s], (it - 1) & 1, abort_flag))) {
          fail(abort_flag, kErrPrefill + 16);
          ok = false;
          break;
        }
#pragma unroll
        for (int ch = 0; ch < 16; ++ch)
          *reinterpret_cast<uint4*>(sm.p[s] + (ch >> 3) * kBoxBytes + sw128_off(row, ch & 7)) =
              make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
        fence_proxy_async_smem();
        mbar_arrive(&sm.pv_ready);
        float s0, s1;
        f2_unpack(f2_add(f2_add(sum2[0], sum2[1]), f2_add(sum2[2], sum2[3])), s0, s1);
        l = l * alpha + (s0 + s1);
        m = m_use;
      }
      if (!ok) break;
      if (it > 0 && !warp_wait(&sm.l_empty[s], (it - 1) & 1, abort_flag)) {
        fail(abort_flag, kErrPrefill + 8);
        break;
      }
      sm.lsum[s][row] = l;
      mbar_arrive(&sm.l_full[s]);
      G += T.n_kv;
    }
  } else {
    // ============================================================ correction
    regs_decrease<kRegsCorrection>();
    const int row = threadIdx.x & (BM - 1);
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    int it = 0, G = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++it) {
      const Tile T = decode_tile<kMode>(a, t);
      const int r = T.r0 + row;  // query row
      // gate logits of this row for both head slots, fetched early
      float glog[2] = {0.f, 0.f};
      if (a.gate && r < a.S) {
        glog[0] = __ldg(a.gate + ((size_t)T.b * a.S + r) * a.Hq + T.h0);
        glog[1] = __ldg(a.gate + ((size_t)T.b * a.S + r) * a.Hq + T.h1);
      }
      for (int j = 0; j < T.n_kv && ok; ++j) {
        for (int s = 0; s < 2; ++s) {
          if (!warp_wait(&sm.alpha_full[s], (G + j) & 1, abort_flag)) {
            fail(abort_flag, kErrPrefill + 9);
            ok = false;
            break;
          }
          const float alpha = sm.alpha[s][row];
          mbar_arrive(&sm.alpha_empty[s]);
          if (j > 0) {
            if (!warp_wait(&sm.pv_done, (G + j - 1) & 1, abort_flag)) {
              fail(abort_flag, kErrPrefill + 10);
              ok = false;
              break;
            }
            tc_fence_after();
            if (__any_sync(0xffffffffu, alpha != 1.f)) {
              const uint32_t oaddr = tmem + lane_off + 256 + s * 128;
#pragma unroll 1
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
          mbar_arrive(&sm.pv_ready);
        }
      }
      if (!ok) break;
      // ---- epilogue: out = O / l * sigmoid(gate), bf16, staged in p[s] for
      // the store warp (P_s(last) is consumed once that slot's P.V is done)
      for (int s = 0; s < 2 && ok; ++s) {
        if (!warp_wait(&sm.pv_done, (G + T.n_kv - 1) & 1, abort_flag) ||
            !warp_wait(&sm.l_full[s], it & 1, abort_flag)) {
          fail(abort_flag, kErrPrefill + 11);
          ok = false;
          break;
        }
        tc_fence_after();
        const float l = sm.lsum[s][row];
        mbar_arrive(&sm.l_empty[s]);
        const float g = a.gate ? 1.f / (1.f + __expf(-glog[s])) : 1.f;
        const float f = g / l;
        uint8_t* stage = sm.p[s];
        const uint32_t oaddr = tmem + lane_off + 256 + s * 128;
#pragma unroll 1
        for (int q4 = 0; q4 < 4; ++q4) {
          uint32_t v[32];
          tmem_ld32(oaddr + q4 * 32, v);
          tmem_wait_ld();
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            const int ch = q4 * 4 + c4;  // 16-byte chunk (8 dims) 0..15
            uint4 u;
            u.x = pack_bf16x2(__uint_as_float(v[8 * c4 + 0]) * f, __uint_as_float(v[8 * c4 + 1]) * f);
            u.y = pack_bf16x2(__uint_as_float(v[8 * c4 + 2]) * f, __uint_as_float(v[8 * c4 + 3]) * f);
            u.z = pack_bf16x2(__uint_as_float(v[8 * c4 + 4]) * f, __uint_as_float(v[8 * c4 + 5]) * f);
            u.w = pack_bf16x2(__uint_as_float(v[8 * c4 + 6]) * f, __uint_as_float(v[8 * c4 + 7]) * f);
            *reinterpret_cast<uint4*>(stage + (ch >> 3) * kBoxBytes + sw128_off(row, ch & 7)) = u;
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(&sm.ost_full[s]);
      }
      G += T.n_kv;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace prefill_detail

namespace prefill_detail {

template <int kMode>
cudaError_t launch_prefill_t(const PrefillArgs& a, const CUtensorMap& q_map, const CUtensorMap& k_map,
                             const CUtensorMap& v_map, const CUtensorMap& o_map, cudaStream_t stream) {
  const long long n_tiles = (long long)a.n_q_tiles * a.n_head_pairs * a.Hkv * a.B;
  if (n_tiles == 0) return cudaSuccess;
  if (n_tiles > 0x7FFFFFFFll) return cudaErrorInvalidConfiguration;
  const size_t smem = sizeof(PrefillSmem);
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
  return launch_kernel(false, prefill_kernel<kMode>, dim3(grid), dim3(kThreads), smem, stream, a, q_map, k_map, v_map,
                          o_map);
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
