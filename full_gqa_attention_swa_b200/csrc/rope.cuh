// Rotary position encoding of Q and K (rotate-half pairs over the first
// rotary_dim dims, angle p * inv_freq[k]: theta^(-2k/rotary_dim), or the
// caller's scaled frequencies), with an optional append
// of the rotated key and the raw value into a KV cache (ring slot p mod W on
// sliding layers, slot p on full layers).
//
// Follows the "Step-3.7-Flash-oQ3e" explainer, section 2.3 (per-layer theta,
// partial rotary on full layers) and section 2.2 (a sliding layer's cache
// keeps the last W tokens), and the "Muse-Glimmer-30B-6bit" explainer's RoPE
// section (theta 0 = no rotation).
//
// Layout of the work: 16 lanes per (token, head) row, one 16-byte chunk of 8
// dims per lane.  A lane reads its chunk and, for rotary dims, the partner
// chunk rotary_dim/2 away, so both halves of a pair are read before any lane
// of the row writes (a __syncwarp separates reads from writes when rotating in
// place).  Each lane forms cos/sin of its 8 frequencies once (see
// rope_cos_sin) and reuses them across all heads it visits.
#pragma once
#include "swa_internal.cuh"

namespace swa {

// calls with at most this many tokens run one block per token
constexpr long long kRopeTokenBlocksMax = 4096;

namespace rope_detail {

constexpr int kChunks = kHeadDim / 8;  // 16-byte chunks per head row

struct Chunk {
  uint4 raw;
};

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
  f[0] = bf16_lo(u.x); f[1] = bf16_hi(u.x);
  f[2] = bf16_lo(u.y); f[3] = bf16_hi(u.y);
  f[4] = bf16_lo(u.z); f[5] = bf16_hi(u.z);
  f[6] = bf16_lo(u.w); f[7] = bf16_hi(u.w);
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  uint4 u;
  u.x = pack_bf16x2(f[0], f[1]);
  u.y = pack_bf16x2(f[2], f[3]);
  u.z = pack_bf16x2(f[4], f[5]);
  u.w = pack_bf16x2(f[6], f[7]);
  return u;
}

// Element e (0..7) of this lane's chunk: its rotary role.
//   role 0: pass-through; role 1: first half (y = x c - x' s);
//   role 2: second half (y = x c + x' s).  freq index k, partner dim.
struct LaneRole {
  int role[8];
  int freq[8];
  int partner[8];
  bool partner_is_chunk;  // partner elements form one aligned chunk
  int partner_chunk;
};

__device__ __forceinline__ LaneRole lane_role(int chunk, int r) {
  LaneRole L;
  const int half = r / 2;
  for (int e = 0; e < 8; ++e) {
    const int d = chunk * 8 + e;
    if (d < half) {
      L.role[e] = 1; L.freq[e] = d; L.partner[e] = d + half;
    } else if (d < r) {
      L.role[e] = 2; L.freq[e] = d - half; L.partner[e] = d - half;
    } else {
      L.role[e] = 0; L.freq[e] = 0; L.partner[e] = d;
    }
  }
  L.partner_is_chunk = (half % 8) == 0 && chunk * 8 < r;
  L.partner_chunk = chunk * 8 < half ? chunk + half / 8 : chunk - half / 8;
  return L;
}

__device__ __forceinline__ void rotate_chunk(const uint16_t* row_src, uint16_t* row_dst, int chunk,
                                             const LaneRole& L, const float (&c)[8], const float (&s)[8],
                                             bool active, bool in_place) {
  uint4 own = make_uint4(0, 0, 0, 0), par = make_uint4(0, 0, 0, 0);
  float xp[8];
  if (active) {
    own = *reinterpret_cast<const uint4*>(row_src + chunk * 8);
    if (L.partner_is_chunk) {
      par = *reinterpret_cast<const uint4*>(row_src + L.partner_chunk * 8);
      unpack8(par, xp);
    } else {
      for (int e = 0; e < 8; ++e) {
        uint32_t b = row_src[L.partner[e]];
        xp[e] = __uint_as_float(b << 16);
      }
    }
  }
  if (in_place) __syncwarp();
  if (active) {
    float x[8], y[8];
    unpack8(own, x);
    for (int e = 0; e < 8; ++e) {
      // one rounding order for every RoPE site: x c + (-/+ x' s), the product x' s rounded first
      if (L.role[e] == 1) y[e] = fmaf(x[e], c[e], -(xp[e] * s[e]));
      else if (L.role[e] == 2) y[e] = fmaf(x[e], c[e], xp[e] * s[e]);
      else y[e] = x[e];
    }
    *reinterpret_cast<uint4*>(row_dst + chunk * 8) = pack8(y);
  }
  if (in_place) __syncwarp();
}

// cos and sin of a rotary angle.  The angle p * inv_freq[k] is formed in
// fp64 and reduced to [-pi, pi] by subtracting the nearest multiple of 2*pi
// (Cody-Waite reduction with 2*pi split into a double and its rounding
// remainder), so its error stays near 1e-15 rad for any position below 2^31;
// the reduced angle is then rounded to fp32 for the hardware sine / cosine
// (__sincosf: absolute error below 1e-6 on [-pi, pi], far under the bf16
// rounding of every rotated value).
__device__ __forceinline__ void rope_cos_sin(double angle, float* c, float* s) {
  const double kTwoPiHi = 6.283185307179586;       // 2*pi rounded to double
  const double kTwoPiLo = 2.4492935982947064e-16;  // 2*pi - kTwoPiHi
  const double n = rint(angle * (1.0 / kTwoPiHi));
  double r = fma(-n, kTwoPiHi, angle);
  r = fma(-n, kTwoPiLo, r);
  __sincosf((float)r, s, c);
}

// grid.x: ceil(B*S*16 / blockDim.x); grid.y: head split (heads h with
// h % gridDim.y == blockIdx.y).  Memory-bound: at least three 256-thread
// blocks per SM keep enough loads in flight (the register cap costs no spill).
__global__ void __launch_bounds__(256, 3) rope_kernel(const RopeArgs a) {
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int chunk = (int)(tid & (kChunks - 1));
  const long long tok = tid >> 4;
  const long long n_tok = (long long)a.B * a.S;
  const bool active = tok < n_tok;
  const long long tk = active ? tok : 0;
  const int b = (int)(tk / a.S);
  const int s_idx = (int)(tk % a.S);
  const int p = a.pos ? a.pos[tk] : a.pos0 + s_idx;

  const int r = a.rotate ? a.rotary_dim : 0;
  const LaneRole L = lane_role(chunk, r);
  float c[8], s[8];
  for (int e = 0; e < 8; ++e) {
    if (L.role[e] != 0) {
      rope_cos_sin((double)p * a.inv_freq[L.freq[e]], &c[e], &s[e]);
    } else {
      c[e] = 1.f;
      s[e] = 0.f;
    }
  }
  if (a.table && active && b == 0 && blockIdx.y == 0) {
    for (int e = 0; e < 8; ++e)
      if (L.role[e] == 1) a.table[rope_table_index(s_idx, L.freq[e], r / 2)] = make_float2(c[e], s[e]);
  }

  const int hs = blockIdx.y, nhs = gridDim.y;
  if (a.q && r > 0) {
    for (int h = hs; h < a.Hq; h += nhs) {
      uint16_t* row = a.q + (tk * a.Hq + h) * kHeadDim;
      rotate_chunk(row, row, chunk, L, c, s, active, true);
    }
  }
  if (a.k_src) {
    const long long dst_tok = (long long)b * (a.dst_rows > 0 ? a.dst_rows : a.S) + a.dst_row_off + s_idx;
    const bool in_place = a.k_dst == a.k_src && dst_tok == tk;
    long long slot = 0;
    bool slot_ok = true;
    if (a.k_cache) {
      slot = a.window > 0 ? (long long)(p % a.window) : (long long)p;
      slot_ok = p >= 0 && slot < a.cache_capacity;
      if (active && !slot_ok && chunk == 0 && hs == 0) record_error(kErrRope + 1);
      if (a.window > 0 && !a.pos) {
        // consecutive positions pos0 .. pos0 + S - 1 on a ring: only the last
        // W are kept, so no two tokens of the call write one slot (explicit
        // positions are the caller's promise of distinct slots)
        slot_ok = slot_ok && p > a.pos0 + a.S - 1 - a.window;
      }
    }
    for (int h = hs; h < a.Hkv; h += nhs) {
      const uint16_t* src = a.k_src + (tk * a.Hkv + h) * kHeadDim;
      uint16_t* dst = a.k_dst + (dst_tok * a.Hkv + h) * kHeadDim;
      if (r > 0 || !in_place) rotate_chunk(src, dst, chunk, L, c, s, active, in_place);
      if (a.k_cache && active && slot_ok) {
        // the rotated chunk: re-read from dst when it was written, else rotate here
        // this lane's own rotated chunk, written above by this same thread
        const uint4 kv = *reinterpret_cast<const uint4*>(dst + chunk * 8);
        uint16_t* kc = a.k_cache + (((long long)b * a.Hkv + h) * a.cache_capacity + slot) * kHeadDim;
        uint16_t* vc = a.v_cache + (((long long)b * a.Hkv + h) * a.cache_capacity + slot) * kHeadDim;
        *reinterpret_cast<uint4*>(kc + chunk * 8) = kv;
        *reinterpret_cast<uint4*>(vc + chunk * 8) =
            *reinterpret_cast<const uint4*>(a.v + (tk * a.Hkv + h) * kHeadDim + chunk * 8);
      }
    }
  }
}

// Keys into a separate buffer, optionally appended with the values to the KV
// cache (the prefill pre-pass, a continued-prefill chunk): the same lanes,
// arithmetic and slot rules as rope_kernel, but every load of the lane's
// heads is issued before the cos/sin and the first store, so a thread waits
// for DRAM once per group of kKeyGroup heads instead of once per head.  With
// rotary_dim / 2 a multiple of 8, a chunk is wholly first half (role 1),
// second half (role 2) or pass-through, and its partner is one whole chunk.
constexpr int kKeyGroup = 8;

__global__ void __launch_bounds__(256, 2) rope_keys_kernel(const RopeArgs a) {
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int chunk = (int)(tid & (kChunks - 1));
  const long long tok = tid >> 4;
  const long long n_tok = (long long)a.B * a.S;
  const bool active = tok < n_tok;
  const long long tk = active ? tok : 0;
  const int b = (int)(tk / a.S);
  const int s_idx = (int)(tk % a.S);
  const int p = a.pos ? a.pos[tk] : a.pos0 + s_idx;
  const int r = a.rotate ? a.rotary_dim : 0;
  const int half = r / 2;
  const int d0 = chunk * 8;
  const int role = d0 < half ? 1 : (d0 < r ? 2 : 0);
  const int k0 = role == 2 ? d0 - half : d0;                 // frequency index of element 0
  const int pchunk = role == 1 ? chunk + half / 8 : chunk - half / 8;
  const long long dst_tok = (long long)b * (a.dst_rows > 0 ? a.dst_rows : a.S) + a.dst_row_off + s_idx;
  const int hs = blockIdx.y, nhs = gridDim.y;
  // cache slot of this token: p mod W on a ring, p on a linear cache
  long long slot = 0;
  bool cache_it = false;
  if (a.k_cache) {
    slot = a.window > 0 ? (long long)(p % a.window) : (long long)p;
    const bool fits = p >= 0 && slot < a.cache_capacity;
    if (active && !fits && chunk == 0 && hs == 0) record_error(kErrRope + 1);
    // consecutive positions on a ring: only the call's last W are kept
    cache_it = active && fits && !(a.window > 0 && !a.pos && p <= a.pos0 + a.S - 1 - a.window);
  }
  bool first = true;
  for (int h0 = hs; h0 < a.Hkv; h0 += nhs * kKeyGroup) {
    uint4 own[kKeyGroup], par[kKeyGroup];
#pragma unroll
    for (int g = 0; g < kKeyGroup; ++g) {
      const int h = h0 + g * nhs;
      own[g] = par[g] = make_uint4(0u, 0u, 0u, 0u);
      if (active && h < a.Hkv) {
        const uint4* src = reinterpret_cast<const uint4*>(a.k_src + (tk * a.Hkv + h) * kHeadDim);
        own[g] = __ldg(src + chunk);
        if (role != 0) par[g] = __ldg(src + pchunk);
      }
    }
    float c[8], sn[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      c[e] = 1.f;
      sn[e] = 0.f;
      if (role != 0) rope_cos_sin((double)p * a.inv_freq[k0 + e], &c[e], &sn[e]);
    }
    if (first && role == 1 && a.table && active && b == 0 && blockIdx.y == 0) {
#pragma unroll
      for (int e = 0; e < 8; ++e) a.table[rope_table_index(s_idx, k0 + e, half)] = make_float2(c[e], sn[e]);
    }
    first = false;
    const float sgn = role == 1 ? -1.f : 1.f;  // y = x c - x' s (first half), x c + x' s (second)
    // (the same rounding order as rope_kernel: the product x' s rounded, then one fma)
#pragma unroll
    for (int g = 0; g < kKeyGroup; ++g) {
      const int h = h0 + g * nhs;
      if (!active || h >= a.Hkv) continue;
      float x[8], xp[8], y[8];
      unpack8(own[g], x);
      unpack8(par[g], xp);
#pragma unroll
      for (int e = 0; e < 8; ++e) y[e] = role == 0 ? x[e] : fmaf(x[e], c[e], sgn * (xp[e] * sn[e]));
      const uint4 yk = pack8(y);
      *reinterpret_cast<uint4*>(a.k_dst + (dst_tok * a.Hkv + h) * kHeadDim + chunk * 8) = yk;
      if (cache_it)
        *reinterpret_cast<uint4*>(a.k_cache + (((long long)b * a.Hkv + h) * a.cache_capacity + slot) * kHeadDim +
                                  chunk * 8) = yk;
    }
    if (cache_it) {  // the raw values follow their keys into the cache
      uint4 vv[kKeyGroup];
#pragma unroll
      for (int g = 0; g < kKeyGroup; ++g) {
        const int h = h0 + g * nhs;
        vv[g] = h < a.Hkv ? __ldg(reinterpret_cast<const uint4*>(a.v + (tk * a.Hkv + h) * kHeadDim) + chunk)
                          : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int g = 0; g < kKeyGroup; ++g) {
        const int h = h0 + g * nhs;
        if (h < a.Hkv)
          *reinterpret_cast<uint4*>(a.v_cache + (((long long)b * a.Hkv + h) * a.cache_capacity + slot) * kHeadDim +
                                    chunk * 8) = vv[g];
      }
    }
  }
}

// One block per token (grid.y: ranges of its heads), for calls with few
// tokens (decode steps, drafts): the block forms the token's cos/sin once
// (shared memory), then every thread
// takes one (head, 16-byte chunk) task per round of 16 heads -- q heads in
// place, then k heads (and the cache append with its value) -- with all loads
// of up to kTokRounds rounds issued before one barrier and all stores after
// it, so rotating in place never reads a chunk another thread already wrote
// (the next batch takes other heads).
// Same arithmetic and slot rules as rope_kernel, so the results are bit for
// bit those of the other paths.  Needs whole partner chunks (rotary_dim / 2 a
// multiple of 8) and writes no cos/sin table.
constexpr int kTokThreads = 256;
constexpr int kTokRounds = 8;  // 8 rounds x 16 heads per load batch

__global__ void __launch_bounds__(kTokThreads) rope_tokens_kernel(const RopeArgs a) {
  allow_dependent_launch();
  grid_dependency_wait();
  __shared__ float2 cs[kMaxRotaryHalf];
  const long long tk = blockIdx.x;
  const int b = (int)(tk / a.S);
  const int s_idx = (int)(tk % a.S);
  const int p = a.pos ? a.pos[tk] : a.pos0 + s_idx;
  const int r = a.rotate ? a.rotary_dim : 0;
  const int half = r / 2;
  if ((int)threadIdx.x < half) {
    float c, sn;
    rope_cos_sin((double)p * a.inv_freq[threadIdx.x], &c, &sn);
    cs[threadIdx.x] = make_float2(c, sn);
  }
  // cache slot of this token: p mod W on a ring, p on a linear cache
  long long slot = 0;
  bool cache_it = false;
  if (a.k_cache) {
    slot = a.window > 0 ? (long long)(p % a.window) : (long long)p;
    const bool fits = p >= 0 && slot < a.cache_capacity;
    if (!fits && threadIdx.x == 0) record_error(kErrRope + 1);
    cache_it = fits && !(a.window > 0 && !a.pos && p <= a.pos0 + a.S - 1 - a.window);
  }
  const long long dst_tok = (long long)b * (a.dst_rows > 0 ? a.dst_rows : a.S) + a.dst_row_off + s_idx;
  const int nq = (a.q && r > 0) ? a.Hq : 0;  // without rotation q is left as it is
  const int nk = a.k_src ? a.Hkv : 0;
  const int chunk = threadIdx.x & (kChunks - 1);
  const int d0 = chunk * 8;
  const int role = d0 < half ? 1 : (d0 < r ? 2 : 0);
  const int k0 = role == 2 ? d0 - half : d0;
  const int pchunk = role == 1 ? chunk + half / 8 : chunk - half / 8;
  const float sgn = role == 1 ? -1.f : 1.f;
  __syncthreads();
  // grid.y splits the token's heads into ranges of whole 16-head rounds
  const int rounds = (nq + nk + kTokThreads / kChunks - 1) / (kTokThreads / kChunks);
  const int per = (rounds + gridDim.y - 1) / gridDim.y;
  const int lo = (int)blockIdx.y * per * (kTokThreads / kChunks);
  const int hi = min(nq + nk, lo + per * (kTokThreads / kChunks));
  for (int base = lo; base < hi; base += kTokRounds * (kTokThreads / kChunks)) {
    uint4 own[kTokRounds], par[kTokRounds], val[kTokRounds];
#pragma unroll
    for (int u = 0; u < kTokRounds; ++u) {
      const int hh = base + u * (kTokThreads / kChunks) + (int)(threadIdx.x / kChunks);  // q heads, then k heads
      own[u] = par[u] = val[u] = make_uint4(0u, 0u, 0u, 0u);
      if (hh < hi) {
        const uint16_t* row = hh < nq ? a.q + (tk * a.Hq + hh) * kHeadDim : a.k_src + (tk * a.Hkv + (hh - nq)) * kHeadDim;
        own[u] = *reinterpret_cast<const uint4*>(row + chunk * 8);
        if (role != 0) par[u] = *reinterpret_cast<const uint4*>(row + pchunk * 8);
        if (hh >= nq && cache_it)
          val[u] = __ldg(reinterpret_cast<const uint4*>(a.v + (tk * a.Hkv + (hh - nq)) * kHeadDim) + chunk);
      }
    }
    __syncthreads();  // every chunk of these heads is read before any is written
#pragma unroll
    for (int u = 0; u < kTokRounds; ++u) {
      const int hh = base + u * (kTokThreads / kChunks) + (int)(threadIdx.x / kChunks);
      if (hh >= hi) continue;
      uint4 yk = own[u];
      if (r > 0 && role != 0) {
        float x[8], xp[8], y[8];
        unpack8(own[u], x);
        unpack8(par[u], xp);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float2 t = cs[k0 + e];
          y[e] = fmaf(x[e], t.x, sgn * (xp[e] * t.y));
        }
        yk = pack8(y);
      }
      if (hh < nq) {
        *reinterpret_cast<uint4*>(a.q + (tk * a.Hq + hh) * kHeadDim + chunk * 8) = yk;
      } else {
        const int h = hh - nq;
        *reinterpret_cast<uint4*>(a.k_dst + (dst_tok * a.Hkv + h) * kHeadDim + chunk * 8) = yk;
        if (cache_it) {
          *reinterpret_cast<uint4*>(a.k_cache + (((long long)b * a.Hkv + h) * a.cache_capacity + slot) * kHeadDim +
                                    chunk * 8) = yk;
          *reinterpret_cast<uint4*>(a.v_cache + (((long long)b * a.Hkv + h) * a.cache_capacity + slot) * kHeadDim +
                                    chunk * 8) = val[u];
        }
      }
    }
  }
}

}  // namespace rope_detail

cudaError_t launch_rope(const RopeArgs& a, cudaStream_t stream) {
  const long long n_tok = (long long)a.B * a.S;
  if (n_tok == 0) return cudaSuccess;
  const int threads = 256;
  const long long lanes = n_tok * rope_detail::kChunks;
  const long long blocks = (lanes + threads - 1) / threads;
  // few tokens (decode): spread heads over grid.y so enough warps run
  int hsplit = 1;
  const int max_heads = a.Hq > a.Hkv ? a.Hq : a.Hkv;
  while (blocks * hsplit < 148 * 4 && hsplit < max_heads) hsplit *= 2;
  if (hsplit > max_heads) hsplit = max_heads;
  if (blocks > 0x7FFFFFFFll) return cudaErrorInvalidConfiguration;
  const int r = a.rotate ? a.rotary_dim : 0;
  if (!a.table && n_tok <= kRopeTokenBlocksMax && ((r / 2) % 8) == 0) {
    // few tokens: spread each token's heads over up to 4 blocks so that about
    // two blocks per SM run
    const int heads = (a.q && r > 0 ? a.Hq : 0) + (a.k_src ? a.Hkv : 0);
    const int rounds = (heads + 15) / 16;
    int ks = 1;
    while (ks < 4 && ks * 2 <= rounds && n_tok * ks < 296) ks *= 2;
    return launch_kernel(true, rope_detail::rope_tokens_kernel, dim3((unsigned)n_tok, (unsigned)ks),
                            dim3(rope_detail::kTokThreads), 0, stream, a);
  }
  const bool keys_only = !a.q && a.k_src && a.k_dst != a.k_src && ((r / 2) % 8) == 0;
  if (keys_only) {
    // one head split while a lane's heads fit one load group: each split
    // recomputes the lane's cos/sin
    const unsigned ks = (unsigned)(a.Hkv <= rope_detail::kKeyGroup ? 1 : hsplit);
    return launch_kernel(false, rope_detail::rope_keys_kernel, dim3((unsigned)blocks, ks), dim3(threads), 0, stream, a);
  }
  return launch_kernel(false, rope_detail::rope_kernel, dim3((unsigned)blocks, (unsigned)hsplit), dim3(threads), 0,
                          stream, a);
}

}  // namespace swa
