// libswa.so: the C ABI declared in include/swa.h.  This file validates
// arguments, plans workspaces and launch shapes, encodes the TMA tensor maps,
// and launches the kernels on the caller's stream.  It is built as a single
// translation unit together with the kernel headers it includes.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <mutex>

#include "../../include/swa.h"
#include "swa_internal.cuh"

#include "decode.cuh"
#include "decode_mq.cuh"
#include "kv_gather.cuh"
#include "prefill.cuh"
#include "rope.cuh"

namespace {

using swa::kHeadDim;

thread_local char g_detail[512] = "";

swa_status fail(swa_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_detail, sizeof g_detail, fmt, ap);
  va_end(ap);
  return st;
}

swa_status ok() {
  g_detail[0] = '\0';
  return SWA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

swa_status check_layer(const swa_layer_params* p) {
  if (!p) return fail(SWA_ERR_INVALID_ARG, "params is NULL");
  if (p->num_q_heads < 1 || p->num_kv_heads < 1)
    return fail(SWA_ERR_INVALID_ARG, "head counts must be >= 1 (Hq=%d, Hkv=%d)", p->num_q_heads, p->num_kv_heads);
  if (p->num_q_heads % p->num_kv_heads != 0)
    return fail(SWA_ERR_INVALID_ARG, "Hq=%d is not a multiple of Hkv=%d", p->num_q_heads, p->num_kv_heads);
  if (p->head_dim <= 0) return fail(SWA_ERR_INVALID_ARG, "head_dim must be positive");
  if (p->head_dim != kHeadDim) return fail(SWA_ERR_UNSUPPORTED, "head_dim=%d (only 128 is supported)", p->head_dim);
  if (p->window == 0 || p->window < -1)
    return fail(SWA_ERR_INVALID_ARG, "window=%d (>= 1, or SWA_WINDOW_FULL)", p->window);
  if (!(p->rope_theta >= 0.0) || !isfinite(p->rope_theta))
    return fail(SWA_ERR_INVALID_ARG, "rope_theta must be finite and >= 0");
  if (p->rotary_dim < 0 || p->rotary_dim > p->head_dim || (p->rotary_dim & 1))
    return fail(SWA_ERR_INVALID_ARG, "rotary_dim=%d (even, 0..head_dim)", p->rotary_dim);
  if (!isfinite(p->softmax_scale)) return fail(SWA_ERR_INVALID_ARG, "softmax_scale is not finite");
  if (p->inv_freq)
    for (int k = 0; k < p->rotary_dim / 2; ++k)
      if (!(p->inv_freq[k] >= 0.0) || !isfinite(p->inv_freq[k]))
        return fail(SWA_ERR_INVALID_ARG, "inv_freq[%d] must be finite and >= 0", k);
  return SWA_OK;
}

// A layer rotates when it has rotary dims and either a frequency table or a
// positive base (theta 0 without a table: no rotary encoding).
bool rotates(const swa_layer_params* p) {
  return p->rotary_dim > 0 && (p->inv_freq != nullptr || p->rope_theta > 0.0);
}

float scale_log2(const swa_layer_params* p) {
  const double s = p->softmax_scale > 0.f ? (double)p->softmax_scale : 1.0 / sqrt((double)p->head_dim);
  return (float)(s * 1.4426950408889634);  // log2(e)
}

void fill_inv_freq(const swa_layer_params* p, double* inv_freq) {
  for (int k = 0; k < swa::kMaxRotaryHalf; ++k) inv_freq[k] = 0.0;
  if (!rotates(p)) return;
  for (int k = 0; k < p->rotary_dim / 2; ++k)
    inv_freq[k] = p->inv_freq ? p->inv_freq[k] : pow(p->rope_theta, -2.0 * (double)k / (double)p->rotary_dim);
}

// ------------------------------------------------------------ TMA encoding

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// bf16 tensor map of rank 3 or 4 with a 128-byte swizzled box whose inner
// extent is 64 elements.  dims/strides as in cuTensorMapEncodeTiled (strides
// in bytes for dims 1..rank-1).
swa_status encode_bf16(CUtensorMap* map, const void* base, int rank, const cuuint64_t* dims,
                       const cuuint64_t* strides, const cuuint32_t* box) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(SWA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SWA_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
  return SWA_OK;
}

// [B, S, H, D] bf16 -> 4-D map {D, H, S, B}, box {64, 1, rows, 1}.
swa_status encode_bshd(CUtensorMap* map, const void* base, int B, int S, int H, int rows) {
  const cuuint64_t dims[4] = {(cuuint64_t)kHeadDim, (cuuint64_t)H, (cuuint64_t)S, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)kHeadDim * 2, (cuuint64_t)H * kHeadDim * 2,
                                 (cuuint64_t)S * H * kHeadDim * 2};
  const cuuint32_t box[4] = {64, 1, (cuuint32_t)rows, 1};
  return encode_bf16(map, base, 4, dims, strides, box);
}

// [B*Hkv, C, D] bf16 cache -> 3-D map {D, keys, B*Hkv} over the first `keys`
// slots (later slots read as zero), box {64, rows, 1}.
swa_status encode_cache_keys(CUtensorMap* map, const void* base, int BH, int C, int keys, int rows) {
  const cuuint64_t dims[3] = {(cuuint64_t)kHeadDim, (cuuint64_t)keys, (cuuint64_t)BH};
  const cuuint64_t strides[2] = {(cuuint64_t)kHeadDim * 2, (cuuint64_t)C * kHeadDim * 2};
  const cuuint32_t box[3] = {64, (cuuint32_t)rows, 1};
  return encode_bf16(map, base, 3, dims, strides, box);
}

// [B*Hkv, C, D] bf16 cache -> 3-D map {D, C, B*Hkv}, box {64, rows, 1}.
swa_status encode_cache(CUtensorMap* map, const void* base, int BH, int C, int rows) {
  const cuuint64_t dims[3] = {(cuuint64_t)kHeadDim, (cuuint64_t)C, (cuuint64_t)BH};
  const cuuint64_t strides[2] = {(cuuint64_t)kHeadDim * 2, (cuuint64_t)C * kHeadDim * 2};
  const cuuint32_t box[3] = {64, (cuuint32_t)rows, 1};
  return encode_bf16(map, base, 3, dims, strides, box);
}

swa_status cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return SWA_OK;
  return fail(SWA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// ------------------------------------------------------------ planning

struct PrefillPlan {
  bool rotate;
  size_t k_bytes, table_bytes, total;
};

PrefillPlan plan_prefill(const swa_layer_params* p, int B, int S) {
  PrefillPlan pl{};
  pl.rotate = rotates(p);
  if (pl.rotate) {
    pl.k_bytes = round_up((size_t)B * S * p->num_kv_heads * kHeadDim * 2, 256);
    pl.table_bytes = round_up((size_t)swa::rope_table_bytes(S, p->rotary_dim / 2), 256);
  }
  pl.total = pl.k_bytes + pl.table_bytes;
  return pl;
}

// Continued prefill: on a ring (sliding) layer the keys / values the chunk
// attends to are assembled in the workspace (h earlier tokens + the chunk);
// on a full layer the chunk is appended to the linear cache first and the
// attention reads the cache in place.
struct ChunkPlan {
  bool rotate, ring;
  int h;  // history rows per sequence (ring)
  size_t k_bytes, v_bytes, table_bytes, total;
};

ChunkPlan plan_prefill_chunk(const swa_layer_params* p, int B, int S, int pos0) {
  ChunkPlan pl{};
  pl.rotate = rotates(p);
  pl.ring = p->window > 0;
  const size_t row = (size_t)p->num_kv_heads * kHeadDim * 2;
  if (pl.ring) {
    pl.h = pos0 < p->window - 1 ? pos0 : p->window - 1;
    pl.k_bytes = round_up((size_t)B * (pl.h + S) * row, 256);
    pl.v_bytes = pl.k_bytes;
  } else if (pl.rotate) {
    pl.k_bytes = round_up((size_t)B * S * row, 256);
  }
  if (pl.rotate) pl.table_bytes = round_up((size_t)swa::rope_table_bytes(S, p->rotary_dim / 2), 256);
  pl.total = pl.k_bytes + pl.v_bytes + pl.table_bytes;
  return pl;
}

struct DecodePlan {
  int chunk, splits;
  size_t o_bytes, ml_bytes, total;
};

DecodePlan plan_decode(const swa_layer_params* p, int B, int max_len) {
  DecodePlan pl{};
  const long long kb = swa::kDecodeKeyBlock;
  const long long n_vis = p->window > 0 ? (max_len < p->window ? max_len : p->window) : max_len;
  // aim for about four resident CTAs per SM (the decode kernel's occupancy)
  // over the whole batch; when the (sequence, kv-head) pairs alone fill at
  // least half of those slots and a whole sequence fits one chunk, splitting
  // would only add waves (and the combine)
  const long long slots = 148 * 4, items = (long long)B * p->num_kv_heads;
  long long c = (items * n_vis + slots - 1) / slots;
  c = (c + kb - 1) / kb * kb;
  if (c < 256) c = 256;
  if (c > 4096) c = 4096;
  if (2 * items >= slots && n_vis <= 4096) c = n_vis;
  if (c >= n_vis) {
    pl.chunk = (int)((n_vis + kb - 1) / kb * kb);
    pl.splits = 1;
  } else {
    pl.chunk = (int)c;
    pl.splits = (int)((n_vis + c - 1) / c);
  }
  if (pl.splits > 1) {
    const size_t rows = (size_t)B * p->num_q_heads * pl.splits;
    pl.o_bytes = round_up(rows * kHeadDim * sizeof(float), 256);
    pl.ml_bytes = round_up(rows * sizeof(float2), 256);
  }
  pl.total = pl.o_bytes + pl.ml_bytes;
  return pl;
}

// Multi-query decode: the same split policy over the cached keys (the new
// tokens ride on the last split), with the kernel's resident CTAs per SM.
DecodePlan plan_decode_mq(const swa_layer_params* p, int B, int T, int max_len) {
  DecodePlan pl{};
  const long long kb = swa::kDecodeMqKeyBlock;
  const long long ctx = max_len - T > 0 ? max_len - T : 0;
  const long long n_vis = p->window > 0 ? (ctx < p->window ? ctx : p->window) : ctx;
  const long long slots = 148LL * swa::kDecodeMqCtasPerSm, items = (long long)B * p->num_kv_heads;
  long long c = (items * n_vis + slots - 1) / slots;
  c = (c + kb - 1) / kb * kb;
  if (c < 256) c = 256;
  if (c > 4096) c = 4096;
  if (2 * items >= slots && n_vis <= 4096) c = n_vis;
  if (c >= n_vis) {
    pl.chunk = (int)(n_vis > 0 ? (n_vis + kb - 1) / kb * kb : kb);
    pl.splits = 1;
  } else {
    pl.chunk = (int)c;
    pl.splits = (int)((n_vis + c - 1) / c);
  }
  if (pl.splits > 1) {
    const size_t rows = (size_t)B * T * p->num_q_heads * pl.splits;
    pl.o_bytes = round_up(rows * kHeadDim * sizeof(float), 256);
    pl.ml_bytes = round_up(rows * sizeof(float2), 256);
  }
  pl.total = pl.o_bytes + pl.ml_bytes;
  return pl;
}

// ------------------------------------------------ no-alloc decode scratch

// Split-K partials of swa_attn_decode_no_alloc.  In host code this name is a
// stand-in, not a device address: the kernels get the address that
// cudaGetSymbolAddress returns for the current device.
static __device__ __align__(256) uint8_t g_decode_scratch[SWA_NO_ALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device, looked up once
// per device (the first call on a device does this).
swa_status scratch_for_current_device(void** ptr) {
  int dev = 0;
  swa_status st = cuda_status(cudaGetDevice(&dev), "cudaGetDevice");
  if (st != SWA_OK) return st;
  if (dev < 0 || dev >= kMaxDevices) return fail(SWA_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    st = cuda_status(cudaGetSymbolAddress(&p, g_decode_scratch), "cudaGetSymbolAddress(decode scratch)");
    if (st != SWA_OK) return st;
    g_scratch_ptr[dev] = p;
  }
  *ptr = g_scratch_ptr[dev];
  return SWA_OK;
}

// The usual decode plan, or -- when its partials exceed the static array --
// the same work in fewer, longer splits, down to one split per row, which
// writes the output directly and needs no scratch at all.
DecodePlan plan_decode_no_alloc(const swa_layer_params* p, int B, int max_len) {
  DecodePlan pl = plan_decode(p, B, max_len);
  if (pl.total <= SWA_NO_ALLOC_SCRATCH_BYTES) return pl;
  const long long kb = swa::kDecodeKeyBlock;
  const long long n_vis = p->window > 0 ? (max_len < p->window ? max_len : p->window) : max_len;
  const size_t rows = (size_t)B * p->num_q_heads;
  const size_t per_split = rows * (kHeadDim * sizeof(float) + sizeof(float2));
  // two 256-byte alignment pads between and after the two arrays
  for (long long fit = (long long)((SWA_NO_ALLOC_SCRATCH_BYTES - 512) / per_split); fit >= 2; --fit) {
    DecodePlan q{};
    q.chunk = (int)(((n_vis + fit - 1) / fit + kb - 1) / kb * kb);
    q.splits = (int)((n_vis + q.chunk - 1) / q.chunk);
    if (q.splits < 2) break;
    q.o_bytes = round_up(rows * q.splits * kHeadDim * sizeof(float), 256);
    q.ml_bytes = round_up(rows * q.splits * sizeof(float2), 256);
    q.total = q.o_bytes + q.ml_bytes;
    if (q.total <= SWA_NO_ALLOC_SCRATCH_BYTES) return q;
  }
  DecodePlan one{};
  one.chunk = (int)((n_vis + kb - 1) / kb * kb);
  one.splits = 1;
  return one;
}

}  // namespace

extern "C" {

const char* swa_version(void) { return "swa-b200 0.1 (sm_100a)"; }

const char* swa_status_string(swa_status s) {
  switch (s) {
    case SWA_OK: return "SWA_OK";
    case SWA_ERR_INVALID_ARG: return "SWA_ERR_INVALID_ARG";
    case SWA_ERR_UNSUPPORTED: return "SWA_ERR_UNSUPPORTED";
    case SWA_ERR_WORKSPACE: return "SWA_ERR_WORKSPACE";
    case SWA_ERR_CUDA: return "SWA_ERR_CUDA";
  }
  return "SWA_ERR_UNKNOWN";
}

const char* swa_last_error_detail(void) { return g_detail; }

swa_status swa_device_error(int32_t* code, int32_t reset) {
  if (!code) return fail(SWA_ERR_INVALID_ARG, "code is NULL");
  swa_status st = cuda_status(cudaDeviceSynchronize(), "cudaDeviceSynchronize");
  if (st != SWA_OK) return st;
  int v = 0;
  st = cuda_status(cudaMemcpyFromSymbol(&v, swa::g_device_error, sizeof(int)), "read device error word");
  if (st != SWA_OK) return st;
  *code = v;
  if (reset) {
    const int zero = 0;
    st = cuda_status(cudaMemcpyToSymbol(swa::g_device_error, &zero, sizeof(int)), "reset device error word");
    if (st != SWA_OK) return st;
  }
  return ok();
}

int64_t swa_kv_cache_bytes(const swa_layer_params* p, int64_t batch, int64_t context) {
  if (check_layer(p) != SWA_OK || batch < 0 || context < 0) return -1;
  const int64_t C = (p->window > 0 && context > p->window) ? p->window : context;
  return batch * p->num_kv_heads * C * p->head_dim * 2 * 2;
}

swa_status swa_rope_qk(const swa_layer_params* p, int32_t B, int32_t S, uint16_t* q, uint16_t* k,
                       const int32_t* pos, int32_t pos0, const uint16_t* v, uint16_t* k_cache, uint16_t* v_cache,
                       int32_t cache_capacity, void* stream) {
  swa_status st = check_layer(p);
  if (st != SWA_OK) return st;
  if (B < 0 || S < 0) return fail(SWA_ERR_INVALID_ARG, "B=%d S=%d must be >= 0", B, S);
  const bool cache = k_cache || v_cache;
  if (cache && !(k_cache && v_cache)) return fail(SWA_ERR_INVALID_ARG, "k_cache and v_cache must both be given");
  if (cache && (!k || !v)) return fail(SWA_ERR_INVALID_ARG, "the cache append needs k and v");
  if (cache) {
    if (cache_capacity < 1) return fail(SWA_ERR_INVALID_ARG, "cache_capacity=%d", cache_capacity);
    if (p->window > 0 && cache_capacity != p->window)
      return fail(SWA_ERR_INVALID_ARG, "sliding layer: cache_capacity=%d must equal window=%d", cache_capacity,
                  p->window);
  }
  if (!pos && pos0 < 0) return fail(SWA_ERR_INVALID_ARG, "pos0=%d must be >= 0", pos0);
  const void* ptrs[] = {q, k, v, k_cache, v_cache, pos};
  for (const void* ptr : ptrs)
    if (ptr && !aligned16(ptr)) return fail(SWA_ERR_INVALID_ARG, "tensor pointer %p is not 16-byte aligned", ptr);
  if ((long long)B * S == 0 || (!q && !k)) return ok();
  if ((long long)B * S * 16 / 256 > 0x7FFFFFFFll) return fail(SWA_ERR_UNSUPPORTED, "too many tokens");
  swa::RopeArgs a{};
  a.B = B; a.S = S; a.Hq = p->num_q_heads; a.Hkv = p->num_kv_heads;
  a.rotary_dim = p->rotary_dim; a.pos0 = pos0; a.pos = pos;
  a.rotate = rotates(p) ? 1 : 0;
  a.q = q; a.k_src = k; a.k_dst = k; a.v = v;
  a.k_cache = k_cache; a.v_cache = v_cache; a.cache_capacity = cache_capacity; a.window = p->window;
  a.table = nullptr;
  fill_inv_freq(p, a.inv_freq);
  if (!a.rotate && !cache) return ok();
  st = cuda_status(swa::launch_rope(a, (cudaStream_t)stream), "rope launch");
  return st == SWA_OK ? ok() : st;
}

size_t swa_prefill_workspace_size(const swa_layer_params* p, int32_t B, int32_t S) {
  if (check_layer(p) != SWA_OK || B < 0 || S < 0) return 0;
  return plan_prefill(p, B, S).total;
}

swa_status swa_attn_prefill(const swa_layer_params* p, int32_t B, int32_t S, const uint16_t* q, const uint16_t* k,
                            const uint16_t* v, const float* gate, uint16_t* out, void* workspace,
                            size_t workspace_bytes, void* stream) {
  swa_status st = check_layer(p);
  if (st != SWA_OK) return st;
  if (B < 0 || S < 0) return fail(SWA_ERR_INVALID_ARG, "B=%d S=%d must be >= 0", B, S);
  if ((long long)B * S == 0) return ok();
  if (!q || !k || !v || !out) return fail(SWA_ERR_INVALID_ARG, "q, k, v and out must be non-NULL");
  const void* ptrs[] = {q, k, v, out, gate, workspace};
  for (const void* ptr : ptrs)
    if (ptr && !aligned16(ptr)) return fail(SWA_ERR_INVALID_ARG, "tensor pointer %p is not 16-byte aligned", ptr);
  const PrefillPlan pl = plan_prefill(p, B, S);
  if (pl.total > 0) {
    if (!workspace) return fail(SWA_ERR_WORKSPACE, "workspace is NULL (%zu bytes needed)", pl.total);
    if (workspace_bytes < pl.total)
      return fail(SWA_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", workspace_bytes, pl.total);
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
      return fail(SWA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  }
  const int Hq = p->num_q_heads, Hkv = p->num_kv_heads, G = Hq / Hkv;
  const long long n_q_tiles = ((long long)S + 127) / 128;
  const long long n_cta = n_q_tiles * ((G + 1) / 2) * Hkv * (long long)B;
  if (n_cta > 0x7FFFFFFFll) return fail(SWA_ERR_UNSUPPORTED, "grid too large (%lld tiles)", n_cta);

  cudaStream_t s = (cudaStream_t)stream;
  const uint16_t* k_att = k;
  float2* table = nullptr;
  if (pl.rotate) {
    uint16_t* k_rot = reinterpret_cast<uint16_t*>(workspace);
    table = reinterpret_cast<float2*>(reinterpret_cast<uint8_t*>(workspace) + pl.k_bytes);
    swa::RopeArgs r{};
    r.B = B; r.S = S; r.Hq = Hq; r.Hkv = Hkv; r.rotary_dim = p->rotary_dim; r.pos0 = 0; r.pos = nullptr;
    r.q = nullptr; r.k_src = k; r.k_dst = k_rot; r.v = nullptr; r.k_cache = nullptr; r.v_cache = nullptr;
    r.cache_capacity = 0; r.window = p->window; r.table = table; r.rotate = 1;
    fill_inv_freq(p, r.inv_freq);
    st = cuda_status(swa::launch_rope(r, s), "rope (keys) launch");
    if (st != SWA_OK) return st;
    k_att = k_rot;
  }
  CUtensorMap qm, km, vm, om;
  if ((st = encode_bshd(&qm, q, B, S, Hq, 128)) != SWA_OK) return st;
  if ((st = encode_bshd(&om, out, B, S, Hq, 128)) != SWA_OK) return st;
  if ((st = encode_bshd(&km, k_att, B, S, Hkv, 128)) != SWA_OK) return st;
  if ((st = encode_bshd(&vm, v, B, S, Hkv, 128)) != SWA_OK) return st;
  swa::PrefillArgs a{};
  a.B = B; a.S = S; a.Hq = Hq; a.Hkv = Hkv; a.G = G; a.window = p->window;
  a.rotary_dim = pl.rotate ? p->rotary_dim : 0;
  a.scale_log2 = scale_log2(p);
  a.table = table;
  a.gate = gate;
  a.n_q_tiles = (int)n_q_tiles;
  a.n_head_pairs = (G + 1) / 2;
  st = cuda_status(swa::launch_prefill(a, qm, km, vm, om, s), "prefill launch");
  return st == SWA_OK ? ok() : st;
}

size_t swa_prefill_chunk_workspace_size(const swa_layer_params* p, int32_t B, int32_t S, int32_t pos0) {
  if (check_layer(p) != SWA_OK || B < 0 || S < 0 || pos0 < 0) return 0;
  return plan_prefill_chunk(p, B, S, pos0).total;
}

swa_status swa_attn_prefill_chunk(const swa_layer_params* p, int32_t B, int32_t S, int32_t pos0, const uint16_t* q,
                                  const uint16_t* k, const uint16_t* v, const float* gate, uint16_t* k_cache,
                                  uint16_t* v_cache, int32_t cache_capacity, uint16_t* out, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  swa_status st = check_layer(p);
  if (st != SWA_OK) return st;
  if (B < 0 || S < 0 || pos0 < 0) return fail(SWA_ERR_INVALID_ARG, "B=%d S=%d pos0=%d must be >= 0", B, S, pos0);
  if ((long long)pos0 + S > 0x7FFFFFFFll) return fail(SWA_ERR_INVALID_ARG, "pos0 + S must stay below 2^31");
  if ((long long)B * S == 0) return ok();
  if (!q || !k || !v || !out || !k_cache || !v_cache)
    return fail(SWA_ERR_INVALID_ARG, "q, k, v, k_cache, v_cache and out must be non-NULL");
  const void* ptrs[] = {q, k, v, out, gate, k_cache, v_cache, workspace};
  for (const void* ptr : ptrs)
    if (ptr && !aligned16(ptr)) return fail(SWA_ERR_INVALID_ARG, "tensor pointer %p is not 16-byte aligned", ptr);
  if (p->window > 0 ? cache_capacity != p->window : (long long)cache_capacity < (long long)pos0 + S)
    return fail(SWA_ERR_INVALID_ARG, "cache_capacity %d: must equal W on a sliding layer, be >= pos0 + S on a full one",
                cache_capacity);
  const ChunkPlan pl = plan_prefill_chunk(p, B, S, pos0);
  if (pl.total > 0) {
    if (!workspace) return fail(SWA_ERR_WORKSPACE, "workspace is NULL (%zu bytes needed)", pl.total);
    if (workspace_bytes < pl.total)
      return fail(SWA_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", workspace_bytes, pl.total);
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
      return fail(SWA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  }
  const int Hq = p->num_q_heads, Hkv = p->num_kv_heads, G = Hq / Hkv;
  const long long n_q_tiles = ((long long)S + 127) / 128;
  if (n_q_tiles * ((G + 1) / 2) * Hkv * (long long)B > 0x7FFFFFFFll)
    return fail(SWA_ERR_UNSUPPORTED, "grid too large");

  cudaStream_t s = (cudaStream_t)stream;
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  uint16_t* k_seq = pl.k_bytes ? reinterpret_cast<uint16_t*>(ws) : nullptr;
  uint16_t* v_seq = pl.v_bytes ? reinterpret_cast<uint16_t*>(ws + pl.k_bytes) : nullptr;
  float2* table = pl.rotate ? reinterpret_cast<float2*>(ws + pl.k_bytes + pl.v_bytes) : nullptr;
  if (pl.ring) {
    // the chunk attends to up to W - 1 earlier tokens: copy them out of the
    // ring before the chunk's own tokens overwrite their slots
    swa::KvGatherArgs g{};
    g.B = B; g.S = S; g.Hkv = Hkv; g.h = pl.h; g.pos0 = pos0; g.window = p->window; g.capacity = cache_capacity;
    g.k_cache = k_cache; g.v_cache = v_cache; g.v = v; g.k_seq = k_seq; g.v_seq = v_seq;
    st = cuda_status(swa::launch_kv_gather(g, s), "history gather launch");
    if (st != SWA_OK) return st;
  }
  // the chunk's keys: rotated at their positions (into the assembled sequence
  // on a ring layer, into scratch on a full one) and, with the values,
  // appended to the cache; the cos/sin table of the chunk's positions
  swa::RopeArgs r{};
  r.B = B; r.S = S; r.Hq = Hq; r.Hkv = Hkv; r.rotary_dim = p->rotary_dim; r.pos0 = pos0; r.pos = nullptr;
  r.q = nullptr; r.k_src = k; r.v = v;
  if (pl.ring) {
    r.k_dst = k_seq; r.dst_rows = pl.h + S; r.dst_row_off = pl.h;
  } else {
    r.k_dst = pl.rotate ? k_seq : const_cast<uint16_t*>(k);  // without rotation nothing is written to k
  }
  r.k_cache = k_cache; r.v_cache = v_cache; r.cache_capacity = cache_capacity; r.window = p->window;
  r.table = table; r.rotate = pl.rotate ? 1 : 0;
  if (pl.rotate) fill_inv_freq(p, r.inv_freq);
  st = cuda_status(swa::launch_rope(r, s), "rope (chunk keys) launch");
  if (st != SWA_OK) return st;

  CUtensorMap qm, km, vm, om;
  if ((st = encode_bshd(&qm, q, B, S, Hq, 128)) != SWA_OK) return st;
  if ((st = encode_bshd(&om, out, B, S, Hq, 128)) != SWA_OK) return st;
  swa::PrefillArgs a{};
  if (pl.ring) {
    if ((st = encode_bshd(&km, k_seq, B, pl.h + S, Hkv, 128)) != SWA_OK) return st;
    if ((st = encode_bshd(&vm, v_seq, B, pl.h + S, Hkv, 128)) != SWA_OK) return st;
    a.q_off = pl.h;
  } else {
    // keys 0 .. pos0 + S - 1 straight from the linear cache
    if ((st = encode_cache_keys(&km, k_cache, B * Hkv, cache_capacity, pos0 + S, 128)) != SWA_OK) return st;
    if ((st = encode_cache_keys(&vm, v_cache, B * Hkv, cache_capacity, pos0 + S, 128)) != SWA_OK) return st;
    a.q_off = pos0;
    a.kv_cache_layout = 1;
  }
  a.B = B; a.S = S; a.Hq = Hq; a.Hkv = Hkv; a.G = G; a.window = p->window;
  a.rotary_dim = pl.rotate ? p->rotary_dim : 0;
  a.scale_log2 = scale_log2(p);
  a.table = table;
  a.gate = gate;
  a.n_q_tiles = (int)n_q_tiles;
  a.n_head_pairs = (G + 1) / 2;
  st = cuda_status(swa::launch_prefill(a, qm, km, vm, om, s), "prefill (chunk) launch");
  return st == SWA_OK ? ok() : st;
}

size_t swa_decode_workspace_size(const swa_layer_params* p, int32_t B, int32_t max_len) {
  if (check_layer(p) != SWA_OK || B < 0 || max_len < 1) return 0;
  return plan_decode(p, B, max_len).total;
}

swa_status swa_attn_decode(const swa_layer_params* p, int32_t B, const uint16_t* q, const float* gate,
                           const uint16_t* k_cache, const uint16_t* v_cache, int32_t cache_capacity,
                           const int32_t* seq_lens, int32_t max_len, uint16_t* out, void* workspace,
                           size_t workspace_bytes, void* stream) {
  swa_status st = check_layer(p);
  if (st != SWA_OK) return st;
  if (B < 0) return fail(SWA_ERR_INVALID_ARG, "B=%d must be >= 0", B);
  if (B == 0) return ok();
  const int Hq = p->num_q_heads, Hkv = p->num_kv_heads, G = Hq / Hkv;
  if (G > 16) return fail(SWA_ERR_UNSUPPORTED, "decode supports up to 16 q-heads per kv-head (G=%d)", G);
  if (!q || !k_cache || !v_cache || !seq_lens || !out)
    return fail(SWA_ERR_INVALID_ARG, "q, k_cache, v_cache, seq_lens and out must be non-NULL");
  const void* ptrs[] = {q, gate, k_cache, v_cache, seq_lens, out, workspace};
  for (const void* ptr : ptrs)
    if (ptr && !aligned16(ptr)) return fail(SWA_ERR_INVALID_ARG, "tensor pointer %p is not 16-byte aligned", ptr);
  if (cache_capacity < 1) return fail(SWA_ERR_INVALID_ARG, "cache_capacity=%d", cache_capacity);
  if (p->window > 0 && cache_capacity != p->window)
    return fail(SWA_ERR_INVALID_ARG, "sliding layer: cache_capacity=%d must equal window=%d", cache_capacity,
                p->window);
  if (max_len < 1) return fail(SWA_ERR_INVALID_ARG, "max_len=%d must be >= 1", max_len);
  if (p->window < 0 && max_len > cache_capacity)
    return fail(SWA_ERR_INVALID_ARG, "full layer: max_len=%d exceeds cache_capacity=%d", max_len, cache_capacity);
  if (B > 65535 || Hkv > 65535) return fail(SWA_ERR_UNSUPPORTED, "B=%d or Hkv=%d too large (grid y / z)", B, Hkv);
  const DecodePlan pl = plan_decode(p, B, max_len);
  if (pl.total > 0) {
    if (!workspace) return fail(SWA_ERR_WORKSPACE, "workspace is NULL (%zu bytes needed)", pl.total);
    if (workspace_bytes < pl.total)
      return fail(SWA_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", workspace_bytes, pl.total);
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
      return fail(SWA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  }
  CUtensorMap km, vm;
  if ((st = encode_cache(&km, k_cache, B * Hkv, cache_capacity, swa::kDecodeKeyBlock)) != SWA_OK) return st;
  if ((st = encode_cache(&vm, v_cache, B * Hkv, cache_capacity, swa::kDecodeKeyBlock)) != SWA_OK) return st;
  swa::DecodeArgs a{};
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.G = G; a.window = p->window; a.capacity = cache_capacity;
  a.scale_log2 = scale_log2(p);
  a.q = q; a.gate = gate; a.seq_lens = seq_lens; a.out = out;
  a.chunk = pl.chunk; a.max_splits = pl.splits;
  a.part_o = pl.splits > 1 ? reinterpret_cast<float*>(workspace) : nullptr;
  a.part_ml = pl.splits > 1 ? reinterpret_cast<float2*>(reinterpret_cast<uint8_t*>(workspace) + pl.o_bytes) : nullptr;
  st = cuda_status(swa::launch_decode(a, km, vm, (cudaStream_t)stream), "decode launch");
  return st == SWA_OK ? ok() : st;
}

size_t swa_decode_mq_workspace_size(const swa_layer_params* p, int32_t B, int32_t T, int32_t max_len) {
  if (check_layer(p) != SWA_OK || B < 0 || T < 1 || T > swa::kDecodeMqMaxT || max_len < T) return 0;
  return plan_decode_mq(p, B, T, max_len).total;
}

swa_status swa_attn_decode_mq(const swa_layer_params* p, int32_t B, int32_t T, const uint16_t* q, const float* gate,
                              const uint16_t* k_new, const uint16_t* v_new, const uint16_t* k_cache,
                              const uint16_t* v_cache, int32_t cache_capacity, const int32_t* seq_lens,
                              int32_t max_len, uint16_t* out, void* workspace, size_t workspace_bytes,
                              void* stream) {
  swa_status st = check_layer(p);
  if (st != SWA_OK) return st;
  if (B < 0) return fail(SWA_ERR_INVALID_ARG, "B=%d must be >= 0", B);
  if (T < 1) return fail(SWA_ERR_INVALID_ARG, "T=%d must be >= 1", T);
  if (B == 0) return ok();
  const int Hq = p->num_q_heads, Hkv = p->num_kv_heads, G = Hq / Hkv;
  if (T > swa::kDecodeMqMaxT || (long long)T * G > swa::kDecodeMqMaxRows)
    return fail(SWA_ERR_UNSUPPORTED, "multi-query decode supports T <= %d and T * G <= %d (T=%d, G=%d)",
                swa::kDecodeMqMaxT, swa::kDecodeMqMaxRows, T, G);
  if (!q || !k_new || !v_new || !k_cache || !v_cache || !seq_lens || !out)
    return fail(SWA_ERR_INVALID_ARG, "q, k_new, v_new, k_cache, v_cache, seq_lens and out must be non-NULL");
  const void* ptrs[] = {q, gate, k_new, v_new, k_cache, v_cache, seq_lens, out, workspace};
  for (const void* ptr : ptrs)
    if (ptr && !aligned16(ptr)) return fail(SWA_ERR_INVALID_ARG, "tensor pointer %p is not 16-byte aligned", ptr);
  if (cache_capacity < 1) return fail(SWA_ERR_INVALID_ARG, "cache_capacity=%d", cache_capacity);
  if (p->window > 0 && cache_capacity != p->window)
    return fail(SWA_ERR_INVALID_ARG, "sliding layer: cache_capacity=%d must equal window=%d", cache_capacity,
                p->window);
  if (max_len < T) return fail(SWA_ERR_INVALID_ARG, "max_len=%d must be >= T=%d", max_len, T);
  if (p->window < 0 && max_len - T > cache_capacity)
    return fail(SWA_ERR_INVALID_ARG, "full layer: max_len - T = %d cached tokens exceed cache_capacity=%d",
                max_len - T, cache_capacity);
  if (B > 65535 || Hkv > 65535) return fail(SWA_ERR_UNSUPPORTED, "B=%d or Hkv=%d too large", B, Hkv);
  const DecodePlan pl = plan_decode_mq(p, B, T, max_len);
  if (pl.total > 0) {
    if (!workspace) return fail(SWA_ERR_WORKSPACE, "workspace is NULL (%zu bytes needed)", pl.total);
    if (workspace_bytes < pl.total)
      return fail(SWA_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", workspace_bytes, pl.total);
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
      return fail(SWA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  }
  // q [B, T, Hq, D] -> {D, Hq, T, B}, box {64, G, T, 1}: the (t, g) rows of one kv-head
  // k_new / v_new [B, T, Hkv, D] -> {D, Hkv, T, B}, box {64, 1, 16, 1} (rows past T read as zero)
  CUtensorMap qm, km, vm, knm, vnm;
  {
    const cuuint64_t dims[4] = {(cuuint64_t)kHeadDim, (cuuint64_t)Hq, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)kHeadDim * 2, (cuuint64_t)Hq * kHeadDim * 2,
                                   (cuuint64_t)T * Hq * kHeadDim * 2};
    const cuuint32_t box[4] = {64, (cuuint32_t)G, (cuuint32_t)T, 1};
    if ((st = encode_bf16(&qm, q, 4, dims, strides, box)) != SWA_OK) return st;
  }
  {
    const cuuint64_t dims[4] = {(cuuint64_t)kHeadDim, (cuuint64_t)Hkv, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)kHeadDim * 2, (cuuint64_t)Hkv * kHeadDim * 2,
                                   (cuuint64_t)T * Hkv * kHeadDim * 2};
    const cuuint32_t box[4] = {64, 1, (cuuint32_t)swa::kDecodeMqMaxT, 1};
    if ((st = encode_bf16(&knm, k_new, 4, dims, strides, box)) != SWA_OK) return st;
    if ((st = encode_bf16(&vnm, v_new, 4, dims, strides, box)) != SWA_OK) return st;
  }
  if ((st = encode_cache(&km, k_cache, B * Hkv, cache_capacity, swa::kDecodeMqKeyBlock)) != SWA_OK) return st;
  if ((st = encode_cache(&vm, v_cache, B * Hkv, cache_capacity, swa::kDecodeMqKeyBlock)) != SWA_OK) return st;
  swa::DecodeMqArgs a{};
  a.B = B; a.T = T; a.Hq = Hq; a.Hkv = Hkv; a.G = G; a.window = p->window; a.capacity = cache_capacity;
  a.scale_log2 = scale_log2(p);
  a.q = q; a.gate = gate; a.k_new = k_new; a.v_new = v_new; a.seq_lens = seq_lens; a.out = out;
  a.chunk = pl.chunk; a.max_splits = pl.splits;
  a.part_o = pl.splits > 1 ? reinterpret_cast<float*>(workspace) : nullptr;
  a.part_ml = pl.splits > 1 ? reinterpret_cast<float2*>(reinterpret_cast<uint8_t*>(workspace) + pl.o_bytes) : nullptr;
  st = cuda_status(swa::launch_decode_mq(a, qm, km, vm, knm, vnm, (cudaStream_t)stream), "multi-query decode launch");
  return st == SWA_OK ? ok() : st;
}

swa_status swa_attn_decode_no_alloc(const swa_layer_params* p, int32_t B, const uint16_t* q, const float* gate,
                                    const uint16_t* k_cache, const uint16_t* v_cache, int32_t cache_capacity,
                                    const int32_t* seq_lens, int32_t max_len, uint16_t* out, void* stream) {
  swa_status st = check_layer(p);
  if (st != SWA_OK) return st;
  if (B < 0) return fail(SWA_ERR_INVALID_ARG, "B=%d must be >= 0", B);
  if (B == 0) return ok();
  const int Hq = p->num_q_heads, Hkv = p->num_kv_heads, G = Hq / Hkv;
  if (G > 16) return fail(SWA_ERR_UNSUPPORTED, "decode supports up to 16 q-heads per kv-head (G=%d)", G);
  if (!q || !k_cache || !v_cache || !seq_lens || !out)
    return fail(SWA_ERR_INVALID_ARG, "q, k_cache, v_cache, seq_lens and out must be non-NULL");
  const void* ptrs[] = {q, gate, k_cache, v_cache, seq_lens, out};
  for (const void* ptr : ptrs)
    if (ptr && !aligned16(ptr)) return fail(SWA_ERR_INVALID_ARG, "tensor pointer %p is not 16-byte aligned", ptr);
  if (cache_capacity < 1) return fail(SWA_ERR_INVALID_ARG, "cache_capacity=%d", cache_capacity);
  if (p->window > 0 && cache_capacity != p->window)
    return fail(SWA_ERR_INVALID_ARG, "sliding layer: cache_capacity=%d must equal window=%d", cache_capacity,
                p->window);
  if (max_len < 1) return fail(SWA_ERR_INVALID_ARG, "max_len=%d must be >= 1", max_len);
  if (p->window < 0 && max_len > cache_capacity)
    return fail(SWA_ERR_INVALID_ARG, "full layer: max_len=%d exceeds cache_capacity=%d", max_len, cache_capacity);
  if (B > 65535 || Hkv > 65535) return fail(SWA_ERR_UNSUPPORTED, "B=%d or Hkv=%d too large (grid y / z)", B, Hkv);
  // the one-time address lookup runs on the first call on a device, whatever
  // that call's plan
  void* scratch = nullptr;
  if ((st = scratch_for_current_device(&scratch)) != SWA_OK) return st;
  const DecodePlan pl = plan_decode_no_alloc(p, B, max_len);
  CUtensorMap km, vm;
  if ((st = encode_cache(&km, k_cache, B * Hkv, cache_capacity, swa::kDecodeKeyBlock)) != SWA_OK) return st;
  if ((st = encode_cache(&vm, v_cache, B * Hkv, cache_capacity, swa::kDecodeKeyBlock)) != SWA_OK) return st;
  swa::DecodeArgs a{};
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.G = G; a.window = p->window; a.capacity = cache_capacity;
  a.scale_log2 = scale_log2(p);
  a.q = q; a.gate = gate; a.seq_lens = seq_lens; a.out = out;
  a.chunk = pl.chunk; a.max_splits = pl.splits;
  a.part_o = pl.splits > 1 ? reinterpret_cast<float*>(scratch) : nullptr;
  a.part_ml = pl.splits > 1 ? reinterpret_cast<float2*>(reinterpret_cast<uint8_t*>(scratch) + pl.o_bytes) : nullptr;
  st = cuda_status(swa::launch_decode(a, km, vm, (cudaStream_t)stream), "decode launch");
  return st == SWA_OK ? ok() : st;
}

}  // extern "C"
