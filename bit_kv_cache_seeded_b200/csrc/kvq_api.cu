// Host side of the kvq C ABI: validation, cache layout, tables, split planning, launches.
// Every entry point validates before launching and reports failures as kvq_status codes.
#include <atomic>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <new>
#include <mutex>
#include <unordered_map>
#include <vector>

#include "kvq_internal.h"
#include "kvq_window.cuh"
#include "kvq_plan.h"

using namespace kvq;

static_assert(kTile * kTilePair == kPlanUnitTokens && kTilePair == kPlanUnitTiles, "split unit = two tiles");

namespace {

constexpr size_t kArenaAlign = 256;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool is_lm_mode(int m) { return m == KVQ_MODE_LM_QJL || m == KVQ_MODE_LM || m == KVQ_MODE_SIGN1; }

kvq_status validate_cfg(const kvq_cfg* c) {
  if (!c) return KVQ_ERR_INVALID_ARG;
  if (c->n_q_heads <= 0 || c->n_kv_heads <= 0 || c->n_q_heads % c->n_kv_heads) return KVQ_ERR_INVALID_ARG;
  if (!(c->softmax_scale >= 0.f) || std::isinf(c->softmax_scale)) return KVQ_ERR_INVALID_ARG;
  if (c->rot_per_head != 0 && c->rot_per_head != 1) return KVQ_ERR_INVALID_ARG;
  if (c->sink_tokens < 0 || c->recent_tokens < 0) return KVQ_ERR_INVALID_ARG;
  if (c->sink_tokens + (long)c->recent_tokens > 1024) return KVQ_ERR_UNSUPPORTED;
  if (c->k_mode == KVQ_MODE_FP4 || c->v_mode == KVQ_MODE_FP4) {
    if (c->rot_per_head) return KVQ_ERR_INVALID_ARG;  // the FP4 latent is not rotated
    if (c->sink_tokens || c->recent_tokens) return KVQ_ERR_UNSUPPORTED;
    if (c->k_mode != KVQ_MODE_FP4 || c->v_mode != KVQ_MODE_FP4) return KVQ_ERR_INVALID_ARG;
    if (c->n_kv_heads != 1) return KVQ_ERR_INVALID_ARG;
    if (c->latent_dim <= 0 || c->rope_dim < 0) return KVQ_ERR_INVALID_ARG;
    if (c->latent_dim != 512 || c->rope_dim != 64) return KVQ_ERR_UNSUPPORTED;
    if (c->n_q_heads != 8 && c->n_q_heads != 16 && c->n_q_heads != 32 && c->n_q_heads != 64)
      return KVQ_ERR_UNSUPPORTED;
    return KVQ_OK;
  }
  if (c->k_mode == KVQ_MODE_KIVI || c->v_mode == KVQ_MODE_KIVI) {
    if (c->k_mode != c->v_mode || c->k_bits != 2 || c->v_bits != 2) return KVQ_ERR_UNSUPPORTED;
    if (c->head_dim != kHeadDim) return c->head_dim > 0 ? KVQ_ERR_UNSUPPORTED : KVQ_ERR_INVALID_ARG;
    if (c->rot_per_head || c->sink_tokens || c->recent_tokens) return KVQ_ERR_INVALID_ARG;
    const int g = c->n_q_heads / c->n_kv_heads;
    if (g != 1 && g != 2 && g != 4 && g != 8) return KVQ_ERR_UNSUPPORTED;
    return KVQ_OK;
  }
  if (!is_lm_mode(c->k_mode) || !is_lm_mode(c->v_mode)) return KVQ_ERR_INVALID_ARG;
  if (c->head_dim != kHeadDim) return c->head_dim > 0 ? KVQ_ERR_UNSUPPORTED : KVQ_ERR_INVALID_ARG;
  const int modes[2] = {c->k_mode, c->v_mode};
  const int bits[2] = {c->k_bits, c->v_bits};
  bool any_qjl = false;
  for (int i = 0; i < 2; ++i) {
    if (modes[i] == KVQ_MODE_SIGN1) {
      if (bits[i] != 1 && bits[i] != 0) return KVQ_ERR_INVALID_ARG;
    } else if (bits[i] < 1 || bits[i] > kMaxBits) {
      return KVQ_ERR_INVALID_ARG;
    }
    any_qjl |= modes[i] == KVQ_MODE_LM_QJL;
  }
  if (any_qjl && c->qjl_dim != kHeadDim) return c->qjl_dim > 0 ? KVQ_ERR_UNSUPPORTED : KVQ_ERR_INVALID_ARG;
  const int g = c->n_q_heads / c->n_kv_heads;
  if (g != 1 && g != 2 && g != 4 && g != 8) return KVQ_ERR_UNSUPPORTED;
  return KVQ_OK;
}

SideLayout make_side(int mode, int bits, int qjl_dim, int order) {
  SideLayout L;
  L.order = order;
  L.bits = (mode == KVQ_MODE_SIGN1) ? 1 : bits;
  L.qjl = mode == KVQ_MODE_LM_QJL;
  L.m = L.qjl ? qjl_dim : 0;
  int off = 0;
  L.off_planes = off;
  off += L.bits * kTile * (kHeadDim / 8);
  L.off_sketch = off;
  off += L.qjl ? kTile * (L.m / 8) : 0;
  L.off_norm = off;
  off += kTile * 2;
  L.off_gamma = off;
  off += L.qjl ? kTile * 2 : 0;
  L.tile_bytes = (int)align_up((size_t)off, 16);
  lloyd_max_f32(L.bits, L.cent, L.thr);
  return L;
}

// KIVI sides: two code bit-planes; keys in octet order with an (unused) norm slot, values in
// byte-lane order with per-token fp16 scale (norm slot) and zero (gamma slot).
SideLayout make_kivi_side(bool values) {
  SideLayout L;
  L.bits = 2;
  L.qjl = 0;
  L.order = values ? kOrderByteLane : kOrderOctet;
  L.off_planes = 0;
  L.off_sketch = 2 * kTile * (kHeadDim / 8);
  L.off_norm = L.off_sketch;
  L.off_gamma = L.off_norm + kTile * 2;
  L.tile_bytes = (int)align_up((size_t)L.off_norm + kTile * 2 * (values ? 2 : 1), 16);
  return L;
}

constexpr int kKiviGroupTokens = 128;  // KIVI key group (four tiles)

Fp4Layout make_fp4(int latent, int rope) {
  Fp4Layout F;
  F.latent = latent;
  F.rope = rope;
  F.off_codes = 0;
  F.off_scales = kTile * latent / 2;
  F.off_rope = F.off_scales + kTile * latent / 16;
  F.tile_bytes = (int)align_up((size_t)F.off_rope + (size_t)kTile * rope * 2, 16);
  return F;
}

struct Plan {
  size_t lens_off, signs_off, S_off, St_off, k_off, v_off, win_off, kstats_off, total;
  bool kivi;
  SideLayout k, v;
  Fp4Layout fp4;
  bool fp4_mode;
  int tiles;
};

// n_pages > 0: a paged cache whose regions are a pool of n_pages pages (two tiles of every kv-head)
// instead of batch x kv-heads x tiles contiguous tiles.
Plan plan_layout(const kvq_cfg* c, int batch, int capacity, int n_pages = 0) {
  Plan P{};
  P.fp4_mode = c->k_mode == KVQ_MODE_FP4;
  P.kivi = c->k_mode == KVQ_MODE_KIVI;
  const int unit = P.kivi ? kKiviGroupTokens : kTile * kTilePair;  // capacity granule
  P.tiles = (capacity + unit - 1) / unit * (unit / kTile);
  size_t off = 0;
  P.lens_off = off;  // lengths, status words, history lengths (window caches)
  off = align_up(off + sizeof(int) * (2 * (size_t)batch + kStatusWords), kArenaAlign);
  const size_t pairs = (size_t)batch * c->n_kv_heads;
  // tiles a region holds: every (sequence, kv-head)'s own, or the page pool's
  const size_t region_tiles = n_pages > 0 ? (size_t)n_pages * c->n_kv_heads * kTilePair : pairs * P.tiles;
  if (P.fp4_mode) {
    P.fp4 = make_fp4(c->latent_dim, c->rope_dim);
    P.signs_off = P.S_off = P.St_off = off;
    P.k_off = off;
    off = align_up(off + region_tiles * (size_t)P.fp4.tile_bytes, kArenaAlign);
    P.v_off = off;
  } else {
    if (P.kivi) {
      P.v = make_kivi_side(true);
      P.k = make_kivi_side(false);
    } else {
      P.v = make_side(c->v_mode, c->v_bits, c->qjl_dim, kOrderByteLane);
      P.k = make_side(c->k_mode, c->k_bits, c->qjl_dim, kOrderToken);
      if (mma_modes_supported(c->n_q_heads / c->n_kv_heads, P.k.bits, P.k.qjl, P.v.bits, P.v.qjl))
        P.k.order = kOrderOctet;
    }
    const size_t m = (P.k.qjl || P.v.qjl) ? (size_t)c->qjl_dim : 0;
    P.signs_off = off;
    off = align_up(off + sizeof(float) * kHeadDim * (c->rot_per_head ? c->n_kv_heads : 1), kArenaAlign);
    P.S_off = off;
    off = align_up(off + sizeof(float) * m * kHeadDim, kArenaAlign);
    P.St_off = off;
    off = align_up(off + sizeof(float) * m * kHeadDim, kArenaAlign);
    P.k_off = off;
    off = align_up(off + region_tiles * (size_t)P.k.tile_bytes, kArenaAlign);
    P.v_off = off;
    off = align_up(off + region_tiles * (size_t)P.v.tile_bytes, kArenaAlign);
    // mixed-precision window (KIVI: the incomplete key group): bf16 K then V, [pairs][slots][d] each
    const size_t slots = P.kivi ? kKiviGroupTokens : (size_t)c->sink_tokens + c->recent_tokens;
    P.win_off = off;
    off = align_up(off + 2 * pairs * slots * kHeadDim * 2, kArenaAlign);
    // KIVI key statistics: [pairs][groups][2][d] fp16
    P.kstats_off = off;
    if (P.kivi) off = align_up(off + pairs * (size_t)(P.tiles / 4) * 2 * kHeadDim * 2, kArenaAlign);
  }
  P.total = off;
  return P;
}

int device_sms() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms > 0 ? sms : 148;
}

// Calls that launch work must run with the cache's device current: its arena, tables and the
// kernels' launches all belong to that device.
bool on_cache_device(const kvq_cache* c) {
  int dev = -1;
  return cudaGetDevice(&dev) == cudaSuccess && dev == c->device;
}

int part_stride(const kvq_cache* c) {
  if (c->is_fp4) return 2 + c->cfg.latent_dim;
  return 2 + kHeadDim * (c->v.qjl ? 2 : 1);
}

// Query prep pieces per (sequence, kv-head) on the tensor-core paths: at most 4 query heads each
// (1 on every other path). The mma.sync kernel also runs one CTA per piece; the tcgen05 kernel
// takes all pieces of a kv-head in one CTA.
int decode_hsplit(const kvq_cache* c) {
  if (c->is_fp4 || c->kivi) return 1;
  const int group = c->cfg.n_q_heads / c->cfg.n_kv_heads;
  if (!mma_modes_supported(group, c->k.bits, c->k.qjl, c->v.bits, c->v.qjl)) return 1;
  return group > 4 ? group / 4 : 1;
}

// Query prep area of one piece of a query group (tensor-core path), and of a whole (sequence,
// kv-head): decode_hsplit pieces.
int prep_piece_stride(const kvq_cache* c) {
  if (c->is_fp4) return 0;
  const int group = c->cfg.n_q_heads / c->cfg.n_kv_heads;
  return mma_prep_bytes(c->k.bits, c->k.qjl, group / decode_hsplit(c));
}
int prep_stride(const kvq_cache* c) { return prep_piece_stride(c) * decode_hsplit(c); }

// Rows of the decode grid the split plan spreads over the SMs: (sequence, kv-head[, piece]).
int decode_rows(const kvq_cache* c) {
  if (c->is_fp4) return c->batch;
  return c->batch * c->cfg.n_kv_heads;  // every LM kernel takes all query heads of a kv-head per CTA
}

size_t partials_bytes(const kvq_cache* c, int splits) {
  return align_up(sizeof(float) * (size_t)c->batch * c->cfg.n_q_heads * splits * part_stride(c), 256);
}

// Workspace = split partials, then the per-(sequence, kv-head) query tables of the tensor-core path.
bool has_window(const kvq_cache* c) { return c->sink > 0 || c->recent > 0 || c->kivi; }

// Bytes of the window's softmax states [B][Hq][parts][part_stride] (window caches), 256-aligned.
size_t window_state_bytes(const kvq_cache* c) {
  if (!has_window(c)) return 0;
  const size_t parts = window_parts(c->sink + c->recent);
  return align_up(sizeof(float) * (size_t)c->batch * c->cfg.n_q_heads * parts * part_stride(c), 256);
}

// Workspace = split partials, the per-(sequence, kv-head) query tables of the tensor-core paths,
// the window's softmax states.
size_t prep_bytes_total(const kvq_cache* c) {
  return align_up((size_t)c->batch * c->cfg.n_kv_heads * prep_stride(c), 256);
}
size_t workspace_for(const kvq_cache* c, int splits) {
  return partials_bytes(c, splits) + prep_bytes_total(c) + window_state_bytes(c);
}

// The lengths the split plan and the split kernels see: the coded history on window caches.
const std::vector<int>& coded_lens(const kvq_cache* c) { return has_window(c) ? c->hlens : c->lens; }

// Resident decode CTAs per SM for a chunk of `units` 64-token units: one for the MLA kernel, the
// tensor-core kernel's shared-memory and register limit for query groups of 1, 2 or 4, else 4.
int decode_slots_per_sm(const kvq_cache* c, int units) {
  if (c->is_fp4 || c->tc || c->kivi_tc) return 1;
  if (c->kivi_cuda) return 8;
  const int group = c->cfg.n_q_heads / c->cfg.n_kv_heads;
  if (group == 1 || group == 2 || group == 4 || group == 8)
    return lm_mma_slots_per_sm(group, c->k, c->v, units * kTile * kTilePair, c->kivi);
  return 4;
}

// Largest chunk (in 64-token units) one decode CTA may take.
int decode_max_units(const kvq_cache* c) {
  if (c->is_fp4) return 1 << 30;
  if (c->tc || c->kivi_tc) return tc_chunk_max(c->cfg.n_q_heads / c->cfg.n_kv_heads) / (kTile * kTilePair);
  if (c->kivi) return kChunkMax / (kTile * kTilePair) / 2 * 2;  // rounded up to whole key groups below
  return kChunkMax / (kTile * kTilePair);
}

// The LM decode kernel a cache uses: the mma.sync kernel (measured faster), or the tcgen05 kernel
// when the environment variable KVQ_DECODE_KERNEL is "tc" (lockstep) or "ws" (warp-specialised) at
// cache creation.
bool choose_tc(const kvq_cfg& cfg, const SideLayout& k, const SideLayout& v) {
  const char* e = std::getenv("KVQ_DECODE_KERNEL");
  if (!e || (std::strcmp(e, "tc") != 0 && std::strcmp(e, "ws") != 0)) return false;
  return k.order == kOrderOctet && tc_modes_supported(cfg.n_q_heads / cfg.n_kv_heads, k.bits, k.qjl, v.bits, v.qjl);
}

// Upper bound on CTAs per SM considered by the split plan (sizes the workspace).
int decode_waves_bound(const kvq_cache* c) { return c->is_fp4 ? 2 : 16; }

float default_scale(const kvq_cfg& cfg) {
  if (cfg.softmax_scale > 0.f) return cfg.softmax_scale;
  const int dqk = (cfg.k_mode == KVQ_MODE_FP4) ? cfg.latent_dim + cfg.rope_dim : cfg.head_dim;
  return 1.0f / std::sqrt((float)dqk);
}

}  // namespace

namespace {
std::atomic<uint64_t> g_launches{0};
thread_local uint64_t t_launches = 0;  // this thread's successful launches (a call's own kernels)
}  // namespace

namespace kvq {
cudaError_t launched() {
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    ++t_launches;
  }
  return e;
}
}  // namespace kvq

extern "C" {

const char* kvq_status_str(kvq_status s) {
  switch (s) {
    case KVQ_OK: return "ok";
    case KVQ_ERR_INVALID_ARG: return "invalid argument";
    case KVQ_ERR_UNSUPPORTED: return "unsupported configuration";
    case KVQ_ERR_CAPACITY: return "cache capacity exceeded";
    case KVQ_ERR_ALIGNMENT: return "misaligned pointer";
    case KVQ_ERR_WORKSPACE: return "buffer too small";
    case KVQ_ERR_CUDA: return "CUDA error";
  }
  return "unknown status";
}

kvq_status kvq_cache_bytes(const kvq_cfg* cfg, int32_t batch, int32_t capacity, size_t* bytes) {
  if (!bytes || batch <= 0 || capacity <= 0) return KVQ_ERR_INVALID_ARG;
  const kvq_status st = validate_cfg(cfg);
  if (st != KVQ_OK) return st;
  *bytes = plan_layout(cfg, batch, capacity).total;
  return KVQ_OK;
}

kvq_status kvq_packed_bytes_per_token(const kvq_cfg* cfg, size_t* bytes) {
  if (!bytes) return KVQ_ERR_INVALID_ARG;
  const kvq_status st = validate_cfg(cfg);
  if (st != KVQ_OK) return st;
  if (cfg->k_mode == KVQ_MODE_FP4) {
    *bytes = (size_t)cfg->latent_dim / 2 + cfg->latent_dim / 16 + 2 * (size_t)cfg->rope_dim;
    return KVQ_OK;
  }
  if (cfg->k_mode == KVQ_MODE_KIVI) {  // per side: codes, plus (K) statistics per 128 tokens or (V) s, z
    *bytes = 2 * ((size_t)cfg->k_bits * kHeadDim / 8 + 4);
    return KVQ_OK;
  }
  size_t b = 0;
  const int modes[2] = {cfg->k_mode, cfg->v_mode}, bits[2] = {cfg->k_bits, cfg->v_bits};
  for (int i = 0; i < 2; ++i) {
    const int nb = modes[i] == KVQ_MODE_SIGN1 ? 1 : bits[i];
    b += (size_t)nb * kHeadDim / 8 + 2;
    if (modes[i] == KVQ_MODE_LM_QJL) b += (size_t)cfg->qjl_dim / 8 + 2;
  }
  *bytes = b;
  return KVQ_OK;
}

kvq_status kvq_cache_bytes_paged(const kvq_cfg* cfg, int32_t batch, int32_t n_pages, size_t* bytes) {
  if (!bytes || batch <= 0 || n_pages <= 0) return KVQ_ERR_INVALID_ARG;
  const kvq_status st = validate_cfg(cfg);
  if (st != KVQ_OK) return st;
  if (cfg->k_mode == KVQ_MODE_FP4) return KVQ_ERR_UNSUPPORTED;
  *bytes = plan_layout(cfg, batch, kTile * kTilePair, n_pages).total;
  return KVQ_OK;
}

}  // extern "C"

namespace {
kvq_status cache_init(kvq_cache** out, const kvq_cfg* cfg, int32_t batch, int32_t capacity, void* dev_mem,
                      size_t dev_bytes, const int8_t* rot_signs, const float* qjl_matrix, void* stream,
                      const int32_t* table, int32_t pages_per_seq, int32_t n_pages) {
  if (!out || !dev_mem || batch <= 0 || capacity <= 0) return KVQ_ERR_INVALID_ARG;
  *out = nullptr;
  const kvq_status st = validate_cfg(cfg);
  if (st != KVQ_OK) return st;
  if (reinterpret_cast<uintptr_t>(dev_mem) % kArenaAlign) return KVQ_ERR_ALIGNMENT;
  if (table && cfg->k_mode == KVQ_MODE_FP4) return KVQ_ERR_UNSUPPORTED;
  const Plan P = plan_layout(cfg, batch, capacity, table ? n_pages : 0);
  if (dev_bytes < P.total) return KVQ_ERR_WORKSPACE;
  const bool need_sketch = !P.fp4_mode && (P.k.qjl || P.v.qjl);
  const int n_signs = P.fp4_mode ? 0 : kHeadDim * (cfg->rot_per_head ? cfg->n_kv_heads : 1);
  // the method's random draws: the caller's arrays, else the configuration's seeds
  std::vector<int8_t> drawn_signs;
  std::vector<float> drawn_S;
  if (!P.fp4_mode && !rot_signs) {
    drawn_signs.resize(n_signs);
    if (kvq_draw_rotation_signs(cfg->rot_seed, n_signs, drawn_signs.data()) != KVQ_OK) return KVQ_ERR_INVALID_ARG;
    rot_signs = drawn_signs.data();
  }
  if (need_sketch && !qjl_matrix) {
    drawn_S.resize((size_t)cfg->qjl_dim * kHeadDim);
    if (kvq_draw_qjl_matrix(cfg->qjl_seed, cfg->qjl_dim, kHeadDim, drawn_S.data()) != KVQ_OK) return KVQ_ERR_INVALID_ARG;
    qjl_matrix = drawn_S.data();
  }
  for (int i = 0; i < n_signs; ++i)
    if (rot_signs[i] != 1 && rot_signs[i] != -1) return KVQ_ERR_INVALID_ARG;

  kvq_cache* c = new (std::nothrow) kvq_cache();
  if (!c) return KVQ_ERR_INVALID_ARG;
  c->cfg = *cfg;
  c->batch = batch;
  c->capacity = P.tiles * kTile;
  c->tiles_per_seq = P.tiles;
  c->dev = static_cast<char*>(dev_mem);
  c->dev_bytes = dev_bytes;
  c->d_lens = reinterpret_cast<int*>(c->dev + P.lens_off);
  c->d_status = c->d_lens + batch;
  c->is_fp4 = P.fp4_mode;
  c->k = P.k;
  c->v = P.v;
  c->fp4 = P.fp4;
  c->d_k = c->dev + P.k_off;
  c->d_v = c->dev + P.v_off;
  c->k_region = P.k_off;
  c->v_region = P.v_off;
  c->lens.assign(batch, 0);
  c->sms = device_sms();
  if (cudaGetDevice(&c->device) != cudaSuccess) {
    delete c;
    return KVQ_ERR_CUDA;
  }
  c->signs_stride = cfg->rot_per_head ? kHeadDim : 0;
  c->tc = !P.fp4_mode && !P.kivi && choose_tc(*cfg, P.k, P.v);
  c->ws = c->tc && std::strcmp(std::getenv("KVQ_DECODE_KERNEL"), "ws") == 0;
  {
    const char* e = std::getenv("KVQ_DECODE_KERNEL");
    // KIVI decode: the mma.sync kernel, or (KVQ_DECODE_KERNEL at cache creation) "tc" the tcgen05
    // kernel, "cuda" the CUDA-core kernel
    c->kivi_tc = P.kivi && e && std::strcmp(e, "tc") == 0;
    c->kivi_cuda = P.kivi && e && std::strcmp(e, "cuda") == 0;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  c->table = table;
  c->pages_per_seq = table ? pages_per_seq : 0;
  c->n_pages = table ? n_pages : 0;
  c->sink = P.fp4_mode ? 0 : cfg->sink_tokens;
  c->recent = P.fp4_mode ? 0 : cfg->recent_tokens;
  c->kivi = P.kivi;
  if (P.kivi) {
    c->recent = kKiviGroupTokens;  // the window slots hold the incomplete last key group
    c->d_kstats = c->dev + P.kstats_off;
    c->groups_per_seq = P.tiles / 4;
  }
  c->d_hlens = c->d_status + kStatusWords;
  c->hlens.assign(batch, 0);
  if (!P.fp4_mode) c->d_win = reinterpret_cast<uint16_t*>(c->dev + P.win_off);
  if (cudaMemsetAsync(c->d_lens, 0, sizeof(int) * (2 * (size_t)batch + kStatusWords), s) != cudaSuccess) {
    delete c;
    return KVQ_ERR_CUDA;
  }
  if (!P.fp4_mode) {
    c->d_signs = reinterpret_cast<float*>(c->dev + P.signs_off);
    c->d_S = reinterpret_cast<float*>(c->dev + P.S_off);
    c->d_St = reinterpret_cast<float*>(c->dev + P.St_off);
    const size_t m = need_sketch ? (size_t)cfg->qjl_dim : 0;
    c->h_tables.resize(n_signs + 2 * m * kHeadDim);
    float* hs = c->h_tables.data();
    for (int i = 0; i < n_signs; ++i) hs[i] = (float)rot_signs[i];
    float* hS = hs + n_signs;
    float* hSt = hS + m * kHeadDim;
    for (size_t j = 0; j < m; ++j)
      for (int i = 0; i < kHeadDim; ++i) {
        hS[j * kHeadDim + i] = qjl_matrix[j * kHeadDim + i];
        hSt[(size_t)i * m + j] = qjl_matrix[j * kHeadDim + i];
      }
    // Synchronous copies: the tables are tiny and this keeps the staging buffer's lifetime
    // trivially safe.
    if (cudaMemcpy(c->d_signs, hs, sizeof(float) * n_signs, cudaMemcpyHostToDevice) != cudaSuccess ||
        (m && cudaMemcpy(c->d_S, hS, sizeof(float) * m * kHeadDim, cudaMemcpyHostToDevice) != cudaSuccess) ||
        (m && cudaMemcpy(c->d_St, hSt, sizeof(float) * m * kHeadDim, cudaMemcpyHostToDevice) != cudaSuccess)) {
      delete c;
      return KVQ_ERR_CUDA;
    }
  }
  *out = c;
  return KVQ_OK;
}
}  // namespace

extern "C" {

kvq_status kvq_cache_init(kvq_cache** out, const kvq_cfg* cfg, int32_t batch, int32_t capacity,
                          void* dev_mem, size_t dev_bytes, const int8_t* rot_signs,
                          const float* qjl_matrix, void* stream) {
  return cache_init(out, cfg, batch, capacity, dev_mem, dev_bytes, rot_signs, qjl_matrix, stream, nullptr, 0, 0);
}

kvq_status kvq_cache_init_paged(kvq_cache** out, const kvq_cfg* cfg, int32_t batch, int32_t pages_per_seq,
                                int32_t n_pages, const int32_t* block_table, void* dev_mem, size_t dev_bytes,
                                const int8_t* rot_signs, const float* qjl_matrix, void* stream) {
  if (!block_table || pages_per_seq <= 0 || n_pages <= 0) return KVQ_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(block_table) % 4) return KVQ_ERR_ALIGNMENT;
  if ((long)pages_per_seq * kTile * kTilePair > (1l << 30)) return KVQ_ERR_INVALID_ARG;
  return cache_init(out, cfg, batch, pages_per_seq * kTile * kTilePair, dev_mem, dev_bytes, rot_signs, qjl_matrix,
                    stream, block_table, pages_per_seq, n_pages);
}

}  // extern "C"

namespace {
// Quantize parameters for sequences [first, first + cnt) of the call (seq_ids may be null: all).
void fill_quantize(QuantizeParams& p, const kvq_cache* c, const void* K, const void* V, kvq_dtype dtype,
                   int n_new, const int32_t* seq_ids, int first, int cnt) {
  const int heads = c->is_fp4 ? 1 : c->cfg.n_kv_heads;
  const size_t elem = dtype == KVQ_BF16 ? 2 : 4;
  const size_t per_seq_k = c->is_fp4 ? (size_t)n_new * c->cfg.latent_dim : (size_t)heads * n_new * kHeadDim;
  const size_t per_seq_v = c->is_fp4 ? (size_t)n_new * c->cfg.rope_dim : per_seq_k;
  std::memset(&p, 0, sizeof(p));
  p.src[0] = static_cast<const char*>(K) + first * per_seq_k * elem;
  p.src[1] = static_cast<const char*>(V) + first * per_seq_v * elem;
  p.bf16 = dtype == KVQ_BF16;
  p.n_new = n_new;
  p.n_seq = cnt;
  p.heads = heads;
  p.region[0] = c->d_k;
  p.region[1] = c->d_v;
  p.tiles_per_seq = c->tiles_per_seq;
  p.table = c->table;
  p.pages_per_seq = c->pages_per_seq;
  p.n_pages = c->n_pages;
  p.side[0] = c->k;
  p.side[1] = c->v;
  p.fp4 = c->fp4;
  p.signs = c->d_signs;
  p.signs_stride = c->signs_stride;
  p.St = c->d_St;
  p.lens = c->d_lens;
  p.err = c->d_status;
  p.wait_limit = kWaitLimitCycles;
  for (int i = 0; i < cnt; ++i) {
    const int sid = seq_ids ? seq_ids[first + i] : first + i;
    p.seq[i] = sid;
    p.pos[i] = c->lens[sid];
  }
}
}  // namespace

namespace {
// Append to a mixed-precision window cache: per launch of up to kMaxSeqPerLaunch sequences, first
// code the tokens that leave the window into the history (from the bf16 ring, or from the input when
// the call appends more tokens than the window holds), then write the new tokens that stay in the
// window. Sequence slots [first, first + cnt) of the call.
kvq_status quantize_window(kvq_cache* c, const void* K, const void* V, kvq_dtype dtype, int n_new,
                           const int32_t* seq_ids, int first, int cnt, cudaStream_t s) {
  QuantizeParams p;
  fill_quantize(p, c, K, V, dtype, n_new, seq_ids, first, cnt);
  const size_t pairs_kv = (size_t)c->batch * c->cfg.n_kv_heads;
  const int slots = c->sink + c->recent;
  p.ring[0] = c->d_win;
  p.ring[1] = c->d_win + pairs_kv * (size_t)slots * kHeadDim;
  p.win_sink = c->sink;
  p.win_recent = c->recent;
  p.win_slots = slots;
  p.src_rows = n_new;
  int max_cnt = 0;
  std::vector<int> h1(cnt);
  for (int i = 0; i < cnt; ++i) {
    const int T0 = c->lens[p.seq[i]], T1 = T0 + n_new;
    const int H0 = std::max(0, T0 - c->recent - c->sink);
    h1[i] = std::max(0, T1 - c->recent - c->sink);
    p.total0[i] = T0;
    p.pos[i] = H0;
    p.cnt[i] = h1[i] - H0;
    max_cnt = std::max(max_cnt, p.cnt[i]);
  }
  if (max_cnt > 0) {  // history appends (reads the ring before the window write below overwrites it)
    QuantizeParams ph = p;
    ph.win_src = 1;
    ph.n_new = max_cnt;
    ph.lens = c->d_hlens;
    // a prefill (every sequence at the same length inside the sink, the same history count) codes
    // its history straight from the input rows after the sink, in whole tiles
    ph.win_input_only = 1;
    ph.src_row0 = c->sink;
    for (int i = 0; i < cnt; ++i)
      if (p.total0[i] != p.total0[0] || p.total0[i] > c->sink || p.cnt[i] != max_cnt) ph.win_input_only = 0;
    if (launch_quantize_lm(ph, 2, s) != cudaSuccess) return KVQ_ERR_CUDA;
    for (int i = 0; i < cnt; ++i) c->hlens[p.seq[i]] = h1[i];
  }
  if (launch_window_write(p, s) != cudaSuccess) return KVQ_ERR_CUDA;
  for (int i = 0; i < cnt; ++i) c->lens[p.seq[i]] += n_new;
  return KVQ_OK;
}
// Append to a KIVI cache: code every 128-token key group the call completes (from the bf16 window
// and the input), then write the call's tokens that are in the new incomplete group to the window.
kvq_status quantize_kivi(kvq_cache* c, const void* K, const void* V, kvq_dtype dtype, int n_new,
                         const int32_t* seq_ids, int first, int cnt, cudaStream_t s) {
  QuantizeParams p;
  fill_quantize(p, c, K, V, dtype, n_new, seq_ids, first, cnt);
  const size_t pairs_kv = (size_t)c->batch * c->cfg.n_kv_heads;
  p.ring[0] = c->d_win;
  p.ring[1] = c->d_win + pairs_kv * (size_t)kKiviGroupTokens * kHeadDim;
  p.win_sink = 0;
  p.win_recent = kKiviGroupTokens;
  p.win_slots = kKiviGroupTokens;
  p.win_kivi = 1;
  p.kstats = c->d_kstats;
  p.groups_per_seq = c->groups_per_seq;
  int max_groups = 0;
  for (int i = 0; i < cnt; ++i) {
    const int T0 = c->lens[p.seq[i]];
    p.total0[i] = T0;
    max_groups = std::max(max_groups, (T0 + n_new) / kKiviGroupTokens - T0 / kKiviGroupTokens);
  }
  if (max_groups > 0) {  // reads the window before the write below overwrites it
    QuantizeParams pg = p;
    pg.lens = c->d_hlens;
    if (launch_kivi_groups(pg, max_groups, s) != cudaSuccess) return KVQ_ERR_CUDA;
  }
  if (launch_window_write(p, s) != cudaSuccess) return KVQ_ERR_CUDA;
  for (int i = 0; i < cnt; ++i) {
    c->lens[p.seq[i]] += n_new;
    c->hlens[p.seq[i]] = c->lens[p.seq[i]] / kKiviGroupTokens * kKiviGroupTokens;
  }
  return KVQ_OK;
}
}  // namespace

extern "C" {

kvq_status kvq_quantize(kvq_cache* c, const void* K, const void* V, kvq_dtype dtype,
                        int32_t n_new, const int32_t* seq_ids, int32_t n_seq, void* stream) {
  if (!c || n_new < 0 || n_seq < 0) return KVQ_ERR_INVALID_ARG;
  if (dtype != KVQ_F32 && dtype != KVQ_BF16) return KVQ_ERR_INVALID_ARG;
  if (n_new == 0 || n_seq == 0) return KVQ_OK;
  if (!K || !V) return KVQ_ERR_INVALID_ARG;
  if (!aligned16(K) || !aligned16(V)) return KVQ_ERR_ALIGNMENT;
  if (!seq_ids && n_seq != c->batch) return KVQ_ERR_INVALID_ARG;
  if (n_seq > c->batch) return KVQ_ERR_INVALID_ARG;
  if (!on_cache_device(c)) return KVQ_ERR_INVALID_ARG;
  std::vector<char> seen(c->batch, 0);
  for (int i = 0; i < n_seq; ++i) {
    const int sid = seq_ids ? seq_ids[i] : i;
    if (sid < 0 || sid >= c->batch || seen[sid]) return KVQ_ERR_INVALID_ARG;
    seen[sid] = 1;
    if ((long)c->lens[sid] + n_new > (long)c->capacity) return KVQ_ERR_CAPACITY;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  for (int first = 0; first < n_seq; first += kMaxSeqPerLaunch) {
    const int cnt = std::min(kMaxSeqPerLaunch, n_seq - first);
    if (c->kivi) {
      const kvq_status st = quantize_kivi(c, K, V, dtype, n_new, seq_ids, first, cnt, s);
      if (st != KVQ_OK) return st;
      continue;
    }
    if (has_window(c)) {
      const kvq_status st = quantize_window(c, K, V, dtype, n_new, seq_ids, first, cnt, s);
      if (st != KVQ_OK) return st;
      continue;
    }
    QuantizeParams p;
    fill_quantize(p, c, K, V, dtype, n_new, seq_ids, first, cnt);
    const cudaError_t e = c->is_fp4 ? launch_quantize_fp4(p, s) : launch_quantize_lm(p, 2, s);
    if (e != cudaSuccess) return KVQ_ERR_CUDA;
    for (int i = 0; i < cnt; ++i) c->lens[p.seq[i]] += n_new;
  }
  return KVQ_OK;
}

kvq_status kvq_workspace_bytes(const kvq_cache* c, size_t* bytes) {
  if (!c || !bytes) return KVQ_ERR_INVALID_ARG;
  const int pairs = decode_rows(c);
  *bytes = workspace_for(c, max_splits(pairs, c->sms, c->tiles_per_seq, decode_max_units(c), decode_waves_bound(c)));
  return KVQ_OK;
}

}  // extern "C"

namespace {
// Shared body of kvq_decode_attention and its test entry (debug_unset_wait: every tensor-core
// decode CTA first waits, bounded by wait_limit cycles, on a barrier that nothing completes).
kvq_status decode_impl(const kvq_cache* c, const void* q, kvq_dtype dtype, float* out, void* workspace,
                       size_t ws_bytes, void* stream, int debug_unset_wait, long long wait_limit,
                       const cudaEvent_t* ev = nullptr, const QuantizeParams* qp = nullptr, float* pout = nullptr) {
  if (!c || !q || (!out && !pout) || !workspace) return KVQ_ERR_INVALID_ARG;
  if (dtype != KVQ_F32 && dtype != KVQ_BF16) return KVQ_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(out ? (const void*)out : (const void*)pout) || !aligned16(workspace))
    return KVQ_ERR_ALIGNMENT;
  if (!on_cache_device(c)) return KVQ_ERR_INVALID_ARG;
  int max_len = 0;
  for (int v : coded_lens(c)) max_len = std::max(max_len, v);
  const int pairs = decode_rows(c);
  int splits, chunk;
  plan_splits(pairs, c->sms, [c](int u) { return decode_slots_per_sm(c, u); }, decode_max_units(c), decode_waves_bound(c), max_len,
              &splits, &chunk);
  if (ws_bytes < workspace_for(c, splits)) return KVQ_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const float log2e = 1.4426950408889634f;
  auto rec = [&](int i) { return !ev || cudaEventRecord(ev[i], s) == cudaSuccess; };
  if (!rec(0)) return KVQ_ERR_CUDA;
  if (c->is_fp4) {
    MlaParams p;
    std::memset(&p, 0, sizeof(p));
    p.q = q;
    p.bf16 = dtype == KVQ_BF16;
    p.out = out;
    p.pout = pout;
    p.part = static_cast<float*>(workspace);
    p.B = c->batch;
    p.Hq = c->cfg.n_q_heads;
    p.splits = splits;
    p.chunk = chunk;
    p.lens = c->d_lens;
    p.reg = c->d_k;
    p.tiles_per_seq = c->tiles_per_seq;
    p.fp4 = c->fp4;
    p.logit_scale = default_scale(c->cfg) * log2e;
    p.err = c->d_status;
    p.wait_limit = wait_limit;
    if (!rec(1) || launch_decode_mla(p, s) != cudaSuccess || !rec(2)) return KVQ_ERR_CUDA;
    if (launch_reduce_mla(p, s) != cudaSuccess || !rec(3)) return KVQ_ERR_CUDA;
    return KVQ_OK;
  }
  DecodeParams p;
  std::memset(&p, 0, sizeof(p));
  p.q = q;
  p.bf16 = dtype == KVQ_BF16;
  p.out = out;
  p.pout = pout;
  p.part = static_cast<float*>(workspace);
  p.part_stride = part_stride(c);
  p.B = c->batch;
  p.Hq = c->cfg.n_q_heads;
  p.Hkv = c->cfg.n_kv_heads;
  p.group = p.Hq / p.Hkv;
  p.splits = splits;
  p.chunk = chunk;
  p.lens = has_window(c) ? c->d_hlens : c->d_lens;
  p.kreg = c->d_k;
  p.vreg = c->d_v;
  p.tiles_per_seq = c->tiles_per_seq;
  p.table = c->table;
  p.pages_per_seq = c->pages_per_seq;
  p.n_pages = c->n_pages;
  p.k = c->k;
  p.v = c->v;
  p.signs = c->d_signs;
  p.signs_stride = c->signs_stride;
  p.S = c->d_S;
  p.St = c->d_St;
  p.logit_scale = default_scale(c->cfg) * log2e;
  p.qprep = static_cast<unsigned char*>(workspace) + partials_bytes(c, splits);
  p.hsplit = decode_hsplit(c);
  p.qprep_stride = prep_piece_stride(c);
  p.err = c->d_status;
  p.wait_limit = wait_limit;
  p.debug_unset_wait = debug_unset_wait;
  p.use_tc = c->tc ? (c->ws ? 2 : 1) : 0;
  if (has_window(c)) {
    const size_t pairs_kv = (size_t)c->batch * c->cfg.n_kv_heads;
    p.wk = c->d_win;
    p.wv = c->d_win + pairs_kv * (size_t)(c->sink + c->recent) * kHeadDim;
    p.win_sink = c->sink;
    p.win_recent = c->recent;
    p.win_slots = c->sink + c->recent;
    p.tot_lens = c->d_lens;
    p.wpart = reinterpret_cast<float*>(static_cast<unsigned char*>(workspace) + partials_bytes(c, splits) +
                                       prep_bytes_total(c));
    p.win_parts = window_parts(p.win_slots);
    p.win_kivi = c->kivi ? 1 : 0;
    p.kstats = c->d_kstats;
    p.groups_per_seq = c->groups_per_seq;
  }
  if (c->kivi) {  // KIVI: the split kernel over the coded groups, the window, the reduce (no rotation)
    if (!c->kivi_cuda && p.chunk % (2 * kTile * kTilePair)) {  // whole 128-token key groups per CTA
      p.chunk += kTile * kTilePair;
      p.splits = std::max(1, (max_len + p.chunk - 1) / p.chunk);
    }
    p.win_fused = !c->kivi_tc && !c->kivi_cuda;  // the mma.sync kernel's extra CTAs take the window
    if (!rec(1)) return KVQ_ERR_CUDA;
    const cudaError_t e = c->kivi_tc ? launch_decode_kivi_tc(p, s)
                          : c->kivi_cuda ? launch_decode_kivi(p, s)
                                         : launch_decode_kivi_mma(p, s);
    if (e != cudaSuccess || !rec(2)) return KVQ_ERR_CUDA;
    if (!p.win_fused && launch_window_decode(p, s) != cudaSuccess) return KVQ_ERR_CUDA;
    if (launch_reduce_lm(p, s) != cudaSuccess || !rec(3)) return KVQ_ERR_CUDA;
    return KVQ_OK;
  }
  const bool tensor_path = p.use_tc ? tc_decode_supported(p) : mma_decode_supported(p);
  if (qp && !tensor_path) {  // no fused front kernel on this path: append first
    if (launch_quantize_lm(*qp, 2, s) != cudaSuccess) return KVQ_ERR_CUDA;
    qp = nullptr;
  }
  p.cache_after_wait = qp != nullptr;
  if (debug_unset_wait && !tensor_path) return KVQ_ERR_UNSUPPORTED;
  p.win_fused = p.wpart && tensor_path && !p.use_tc;  // the mma.sync split kernel takes the window parts
  if (launch_decode_lm(p, s, ev ? ev[1] : nullptr, qp) != cudaSuccess || !rec(2)) return KVQ_ERR_CUDA;
  if (p.wpart && !p.win_fused && launch_window_decode(p, s) != cudaSuccess) return KVQ_ERR_CUDA;
  if (launch_reduce_lm(p, s) != cudaSuccess || !rec(3)) return KVQ_ERR_CUDA;
  return KVQ_OK;
}
}  // namespace

extern "C" {

kvq_status kvq_decode_attention(const kvq_cache* c, const void* q, kvq_dtype dtype, float* out,
                                void* workspace, size_t ws_bytes, void* stream) {
  return decode_impl(c, q, dtype, out, workspace, ws_bytes, stream, 0, kWaitLimitCycles);
}

kvq_status kvq_partial_floats(const kvq_cache* c, int32_t* floats) {
  if (!c || !floats) return KVQ_ERR_INVALID_ARG;
  *floats = 2 + (c->is_fp4 ? c->cfg.latent_dim : kHeadDim);
  return KVQ_OK;
}

kvq_status kvq_decode_partials(const kvq_cache* c, const void* q, kvq_dtype dtype, float* partials,
                               void* workspace, size_t ws_bytes, void* stream) {
  if (!partials) return KVQ_ERR_INVALID_ARG;
  return decode_impl(c, q, dtype, nullptr, workspace, ws_bytes, stream, 0, kWaitLimitCycles, nullptr, nullptr,
                     partials);
}

kvq_status kvq_combine_partials(const float* partials, int32_t n_parts, int32_t batch, int32_t n_q_heads,
                                int32_t dv, float* out, void* stream) {
  if (!partials || !out || n_parts < 1 || batch < 1 || n_q_heads < 1 || dv < 1) return KVQ_ERR_INVALID_ARG;
  if (!aligned16(partials) || !aligned16(out)) return KVQ_ERR_ALIGNMENT;
  const long rows = (long)batch * n_q_heads;
  if (rows > (1l << 31) - 1) return KVQ_ERR_INVALID_ARG;
  return launch_combine_partials(partials, n_parts, (int)rows, dv, out, reinterpret_cast<cudaStream_t>(stream)) ==
                 cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

kvq_status kvq_decode_step(kvq_cache* c, const void* K, const void* V, const void* q, kvq_dtype dtype,
                           float* out, void* workspace, size_t ws_bytes, void* stream) {
  if (!c || !K || !V || !q || !out || !workspace) return KVQ_ERR_INVALID_ARG;
  if (dtype != KVQ_F32 && dtype != KVQ_BF16) return KVQ_ERR_INVALID_ARG;
  if (!aligned16(K) || !aligned16(V) || !aligned16(q) || !aligned16(out) || !aligned16(workspace))
    return KVQ_ERR_ALIGNMENT;
  if (!on_cache_device(c)) return KVQ_ERR_INVALID_ARG;
  // everything both halves check, with the lengths after the append, before anything is written
  int max_len = 0;
  for (int v : c->lens) {
    if ((long)v + 1 > (long)c->capacity) return KVQ_ERR_CAPACITY;
  }
  for (int v : coded_lens(c)) max_len = std::max(max_len, v);
  const int pairs = decode_rows(c);
  int splits, chunk;
  plan_splits(pairs, c->sms, [c](int u) { return decode_slots_per_sm(c, u); }, decode_max_units(c), decode_waves_bound(c), max_len + 1,
              &splits, &chunk);
  if (ws_bytes < workspace_for(c, splits)) return KVQ_ERR_WORKSPACE;
  if (c->is_fp4 || c->batch > kMaxSeqPerLaunch || has_window(c)) {  // no fused front kernel: the two calls in sequence
    const kvq_status st = kvq_quantize(c, K, V, dtype, 1, nullptr, c->batch, stream);
    if (st != KVQ_OK) return st;
    return decode_impl(c, q, dtype, out, workspace, ws_bytes, stream, 0, kWaitLimitCycles);
  }
  QuantizeParams qp;
  fill_quantize(qp, c, K, V, dtype, 1, nullptr, 0, c->batch);
  for (int i = 0; i < c->batch; ++i) c->lens[i] += 1;  // the plan of the decode sees the new lengths
  const uint64_t launches0 = t_launches;
  const kvq_status st = decode_impl(c, q, dtype, out, workspace, ws_bytes, stream, 0, kWaitLimitCycles, nullptr, &qp);
  // The append is the step's first kernel: if nothing was launched, nothing was appended and the
  // host lengths go back. (A failure of a later kernel leaves the append enqueued.)
  if (st != KVQ_OK && t_launches == launches0)
    for (int i = 0; i < c->batch; ++i) c->lens[i] -= 1;
  return st;
}

}  // extern "C"

namespace {
// Byte sizes of one step's K, V, q and out, and their offsets in the staging buffer: two input
// slots (K, V, q each), then two output slots.
struct StepStaging {
  size_t n[4] = {};    // K, V, q, out
  size_t off[4] = {};  // within an input slot (out: the first output slot, within the buffer)
  size_t slot = 0;     // bytes of one input slot
  size_t out_slot = 0; // bytes of one output slot
  size_t total = 0;
};
StepStaging step_staging(const kvq_cache* c, kvq_dtype dtype) {
  const size_t elem = dtype == KVQ_BF16 ? 2 : 4, B = (size_t)c->batch, Hq = (size_t)c->cfg.n_q_heads;
  StepStaging S;
  if (c->is_fp4) {
    S.n[0] = B * c->cfg.latent_dim * elem;
    S.n[1] = B * c->cfg.rope_dim * elem;
    S.n[2] = B * Hq * (size_t)(c->cfg.latent_dim + c->cfg.rope_dim) * elem;
    S.n[3] = B * Hq * (size_t)c->cfg.latent_dim * sizeof(float);
  } else {
    S.n[0] = S.n[1] = B * (size_t)c->cfg.n_kv_heads * kHeadDim * elem;
    S.n[2] = B * Hq * kHeadDim * elem;
    S.n[3] = B * Hq * kHeadDim * sizeof(float);
  }
  for (int i = 0; i < 3; ++i) {
    S.off[i] = S.slot;
    S.slot = align_up(S.slot + S.n[i], 256);
  }
  S.off[3] = 2 * S.slot;
  S.out_slot = align_up(S.n[3], 256);
  S.total = S.off[3] + 2 * S.out_slot;
  return S;
}

// Per cache: the two copy streams of kvq_decode_step_host (host -> device inputs, device -> host
// output) and, per slot, the events "inputs landed" (input stream), "step done" (caller's stream)
// and "output copied" (output stream). Created at the first call, released by kvq_cache_destroy.
struct HostStep {
  cudaStream_t copy = nullptr, copy_out = nullptr;
  cudaEvent_t landed[2] = {}, done[2] = {}, copied[2] = {};
  unsigned long long calls = 0;
};
std::mutex g_host_step_mu;
std::unordered_map<const kvq_cache*, HostStep> g_host_step;

void release_host_step(HostStep& h) {
  for (int i = 0; i < 2; ++i) {
    if (h.landed[i]) cudaEventDestroy(h.landed[i]);
    if (h.done[i]) cudaEventDestroy(h.done[i]);
    if (h.copied[i]) cudaEventDestroy(h.copied[i]);
  }
  if (h.copy) cudaStreamDestroy(h.copy);
  if (h.copy_out) cudaStreamDestroy(h.copy_out);
  h = HostStep{};
}

HostStep* host_step_state(const kvq_cache* c) {
  std::lock_guard<std::mutex> lock(g_host_step_mu);
  HostStep& h = g_host_step[c];
  if (h.copy) return &h;
  bool ok = cudaStreamCreateWithFlags(&h.copy, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&h.copy_out, cudaStreamNonBlocking) == cudaSuccess;
  for (int i = 0; i < 2 && ok; ++i)
    ok = cudaEventCreateWithFlags(&h.landed[i], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&h.done[i], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&h.copied[i], cudaEventDisableTiming) == cudaSuccess;
  if (ok) return &h;
  release_host_step(h);
  g_host_step.erase(c);
  return nullptr;
}

void forget_host_step(const kvq_cache* c) {
  std::lock_guard<std::mutex> lock(g_host_step_mu);
  auto it = g_host_step.find(c);
  if (it == g_host_step.end()) return;
  release_host_step(it->second);
  g_host_step.erase(it);
}
}  // namespace

extern "C" {

kvq_status kvq_step_staging_bytes(const kvq_cache* c, kvq_dtype dtype, size_t* bytes) {
  if (!c || !bytes || (dtype != KVQ_F32 && dtype != KVQ_BF16)) return KVQ_ERR_INVALID_ARG;
  *bytes = step_staging(c, dtype).total;
  return KVQ_OK;
}

kvq_status kvq_decode_step_host(kvq_cache* c, const void* K, const void* V, const void* q, kvq_dtype dtype,
                                float* out, void* staging, size_t staging_bytes, void* workspace,
                                size_t ws_bytes, void* stream, void* out_event) {
  if (!c || !K || !V || !q || !out || !staging || !workspace) return KVQ_ERR_INVALID_ARG;
  if (dtype != KVQ_F32 && dtype != KVQ_BF16) return KVQ_ERR_INVALID_ARG;
  if (!aligned16(staging) || !aligned16(workspace)) return KVQ_ERR_ALIGNMENT;
  const StepStaging S = step_staging(c, dtype);
  if (staging_bytes < S.total) return KVQ_ERR_INVALID_ARG;
  // what kvq_decode_step would refuse, refused before any copy
  int max_len = 0;
  for (int v : c->lens)
    if ((long)v + 1 > (long)c->capacity) return KVQ_ERR_CAPACITY;
  for (int v : coded_lens(c)) max_len = std::max(max_len, v);
  int splits, chunk;
  plan_splits(decode_rows(c), c->sms, [c](int u) { return decode_slots_per_sm(c, u); }, decode_max_units(c),
              decode_waves_bound(c), max_len + 1, &splits, &chunk);
  if (ws_bytes < workspace_for(c, splits)) return KVQ_ERR_WORKSPACE;
  HostStep* h = host_step_state(c);
  if (!h) return KVQ_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int slot = (int)(h->calls & 1);
  char* in = static_cast<char*>(staging) + slot * S.slot;
  char* dout = static_cast<char*>(staging) + S.off[3] + slot * S.out_slot;
  // the inputs cross on the input stream once the step two calls back has read this slot, while
  // the previous step may still run; the step waits for them on the caller's stream, and for the
  // output copy of the step two calls back to have left this output slot
  if (cudaStreamWaitEvent(h->copy, h->done[slot], 0) != cudaSuccess) return KVQ_ERR_CUDA;
  const void* src[3] = {K, V, q};
  for (int i = 0; i < 3; ++i)
    if (cudaMemcpyAsync(in + S.off[i], src[i], S.n[i], cudaMemcpyHostToDevice, h->copy) != cudaSuccess)
      return KVQ_ERR_CUDA;
  if (cudaEventRecord(h->landed[slot], h->copy) != cudaSuccess || cudaStreamWaitEvent(s, h->landed[slot], 0) != cudaSuccess ||
      cudaStreamWaitEvent(s, h->copied[slot], 0) != cudaSuccess)
    return KVQ_ERR_CUDA;
  const kvq_status r = kvq_decode_step(c, in + S.off[0], in + S.off[1], in + S.off[2], dtype,
                                       reinterpret_cast<float*>(dout), workspace, ws_bytes, stream);
  if (r != KVQ_OK) return r;
  ++h->calls;
  // the output leaves on the output stream, overlapping the caller's next step
  if (cudaEventRecord(h->done[slot], s) != cudaSuccess || cudaStreamWaitEvent(h->copy_out, h->done[slot], 0) != cudaSuccess ||
      cudaMemcpyAsync(out, dout, S.n[3], cudaMemcpyDeviceToHost, h->copy_out) != cudaSuccess ||
      cudaEventRecord(h->copied[slot], h->copy_out) != cudaSuccess)
    return KVQ_ERR_CUDA;
  if (out_event) return cudaEventRecord(static_cast<cudaEvent_t>(out_event), h->copy_out) == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
  return cudaStreamWaitEvent(s, h->copied[slot], 0) == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

kvq_status kvq_debug_decode_unset_wait(const kvq_cache* c, const void* q, kvq_dtype dtype, float* out,
                                       void* workspace, size_t ws_bytes, int64_t wait_limit_cycles,
                                       void* stream) {
  if (wait_limit_cycles <= 0 || wait_limit_cycles > kWaitLimitCycles) return KVQ_ERR_INVALID_ARG;
  return decode_impl(c, q, dtype, out, workspace, ws_bytes, stream, 1, wait_limit_cycles);
}

kvq_status kvq_debug_decode_timed(const kvq_cache* c, const void* q, kvq_dtype dtype, float* out,
                                  void* workspace, size_t ws_bytes, void* stream, void* const* events) {
  if (!events || !events[0] || !events[1] || !events[2] || !events[3]) return KVQ_ERR_INVALID_ARG;
  cudaEvent_t ev[4];
  for (int i = 0; i < 4; ++i) ev[i] = static_cast<cudaEvent_t>(events[i]);
  return decode_impl(c, q, dtype, out, workspace, ws_bytes, stream, 0, kWaitLimitCycles, ev);
}

kvq_status kvq_cache_status(const kvq_cache* c, int32_t* status, void* stream) {
  if (!c || !status) return KVQ_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(status, c->d_status, sizeof(int32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return KVQ_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return KVQ_ERR_CUDA;
  return KVQ_OK;
}

uint64_t kvq_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

kvq_status kvq_cache_lengths(const kvq_cache* c, int32_t* lens) {
  if (!c || !lens) return KVQ_ERR_INVALID_ARG;
  for (int i = 0; i < c->batch; ++i) lens[i] = c->lens[i];
  return KVQ_OK;
}

kvq_status kvq_cache_layout(const kvq_cache* c, int64_t* info, int32_t n_info) {
  if (!c || !info || n_info < 16) return KVQ_ERR_INVALID_ARG;
  if (n_info > 16) info[16] = c->is_fp4 ? 0 : c->k.order;
  if (n_info > 17) info[17] = c->is_fp4 ? 0 : c->v.order;
  for (int i = 18; i < n_info; ++i) info[i] = 0;
  if (n_info > 21) {
    info[18] = c->d_win ? (int64_t)(reinterpret_cast<char*>(c->d_win) - c->dev) : 0;
    info[19] = c->sink + c->recent;
    info[20] = c->sink;
    info[21] = c->recent;
  }
  if (n_info > 23) {
    info[22] = c->pages_per_seq;
    info[23] = c->n_pages;
  }
  info[0] = kTile;
  info[1] = c->is_fp4 ? c->fp4.tile_bytes : c->k.tile_bytes;
  info[2] = c->is_fp4 ? 0 : c->v.tile_bytes;
  info[3] = c->tiles_per_seq;
  info[4] = (int64_t)c->k_region;
  info[5] = (int64_t)c->v_region;
  if (c->is_fp4) {
    info[6] = c->fp4.off_codes;
    info[7] = c->fp4.off_scales;
    info[8] = c->fp4.off_rope;
    for (int i = 9; i < 16; ++i) info[i] = 0;
    return KVQ_OK;
  }
  const SideLayout* sides[2] = {&c->k, &c->v};
  for (int i = 0; i < 2; ++i) {
    info[6 + 5 * i] = sides[i]->off_planes;
    info[7 + 5 * i] = sides[i]->off_sketch;
    info[8 + 5 * i] = sides[i]->off_norm;
    info[9 + 5 * i] = sides[i]->off_gamma;
    info[10 + 5 * i] = sides[i]->bits;
  }
  return KVQ_OK;
}

kvq_status kvq_lloyd_max_table(int32_t bits, float* centroids, float* thresholds) {
  if (bits < 1 || bits > kMaxBits || !centroids || !thresholds) return KVQ_ERR_INVALID_ARG;
  lloyd_max_f32(bits, centroids, thresholds);
  return KVQ_OK;
}

void kvq_cache_destroy(kvq_cache* c) {
  if (!c) return;
  forget_host_step(c);
  delete c;
}

kvq_status kvq_debug_quantize_rotated(const kvq_cache* c, const float* u, int32_t n,
                                      uint32_t* planes, uint32_t* sketch, uint16_t* gamma,
                                      void* stream) {
  if (!c || c->is_fp4 || n < 0) return KVQ_ERR_INVALID_ARG;
  if (n == 0) return KVQ_OK;
  if (!u || !planes || (c->k.qjl && (!sketch || !gamma))) return KVQ_ERR_INVALID_ARG;
  if (!aligned16(u) || !aligned16(planes) || (sketch && !aligned16(sketch))) return KVQ_ERR_ALIGNMENT;
  QuantizeParams p;
  std::memset(&p, 0, sizeof(p));
  p.src[0] = u;
  p.bf16 = 0;
  p.n_new = n;
  p.n_seq = 1;
  p.heads = 1;
  p.side[0] = c->k;
  p.signs = c->d_signs;
  p.St = c->d_St;
  p.err = c->d_status;
  p.wait_limit = kWaitLimitCycles;
  p.skip_rotation = 1;
  p.dbg_planes = planes;
  p.dbg_sketch = sketch;
  p.dbg_gamma = gamma;
  if (launch_quantize_lm(p, 1, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return KVQ_ERR_CUDA;
  return KVQ_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------------------------
// Allocation-free decode entry point.
//
// Some callers cannot hand the library a workspace: serving loops that reserve all device
// memory at start-up and forbid any further allocation on the decode path, hosts whose device
// memory belongs to another allocator, and code that must not call cudaMalloc because it can
// synchronize the device. For them kvq_decode_attention_static keeps the split-K partials in
// the fixed array below instead of a caller workspace.
//
// The array is file-scope device memory: every GPU that loads this library holds its 16 MiB
// until the process exits. Its address is a device address only on the device side; host code
// gets it from cudaGetSymbolAddress with the cache's device current. A call outside stream
// capture looks the address up again (a context that was reset and re-created reloads the module,
// and the array may move); a call on a capturing stream, which may not trigger a module load, uses
// the address the last uncaptured call on that device found. Nothing in it has to start at zero:
// each call writes every partial slot it later reads. All calls share it, so two calls that
// overlap on the GPU (e.g. on different streams) race.
// ---------------------------------------------------------------------------------------------

namespace {
constexpr size_t kStaticScratchBytes = size_t(16) << 20;
constexpr int kMaxDevices = 64;
std::mutex g_static_scratch_mu;
void* g_static_scratch_ptr[kMaxDevices] = {};
}  // namespace

static __device__ __align__(256) float g_kvq_static_scratch[kStaticScratchBytes / sizeof(float)];

namespace {
kvq_status static_scratch_for_current_device(cudaStream_t s, void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return KVQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return KVQ_ERR_UNSUPPORTED;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cap) != cudaSuccess) return KVQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_static_scratch_mu);
  if (cap == cudaStreamCaptureStatusNone) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_kvq_static_scratch) != cudaSuccess || !p) return KVQ_ERR_CUDA;
    g_static_scratch_ptr[dev] = p;
  } else if (!g_static_scratch_ptr[dev]) {
    return KVQ_ERR_CUDA;  // no uncaptured call has looked the address up on this device yet
  }
  *out = g_static_scratch_ptr[dev];
  return KVQ_OK;
}
}  // namespace

extern "C" kvq_status kvq_decode_attention_static(const kvq_cache* c, const void* q, kvq_dtype dtype,
                                                  float* out, void* stream) {
  if (!c || !q || !out) return KVQ_ERR_INVALID_ARG;
  if (!on_cache_device(c)) return KVQ_ERR_INVALID_ARG;
  int max_len = 0;
  for (int v : coded_lens(c)) max_len = std::max(max_len, v);
  const int pairs = decode_rows(c);
  int splits, chunk;
  plan_splits(pairs, c->sms, [c](int u) { return decode_slots_per_sm(c, u); }, decode_max_units(c), decode_waves_bound(c), max_len,
              &splits, &chunk);
  if (workspace_for(c, splits) > kStaticScratchBytes) return KVQ_ERR_WORKSPACE;
  void* scratch = nullptr;
  const kvq_status st = static_scratch_for_current_device(reinterpret_cast<cudaStream_t>(stream), &scratch);
  if (st != KVQ_OK) return st;
  return kvq_decode_attention(c, q, dtype, out, scratch, kStaticScratchBytes, stream);
}
