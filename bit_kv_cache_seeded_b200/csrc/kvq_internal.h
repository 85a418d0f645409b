// Internal definitions shared by the host API and the kernels of the kvq library.
#pragma once

#include <cstddef>
#include <cstdint>
#include <vector>

#include <cuda_runtime.h>

#include "kvq.h"

namespace kvq {

constexpr int kTile = 32;          // tokens per cache tile
constexpr int kHeadDim = 128;      // head_dim supported by the rotated (LM/SIGN1) modes
constexpr int kMaxSeqPerLaunch = 1024;
constexpr int kMaxBits = 3;
constexpr int kTilePair = 2;      // cache tiles are allocated and split in pairs (64 tokens)
constexpr int kChunkMax = 2240;   // largest context chunk of one decode CTA (LM tensor-core path): its
                                  // logits still leave room for four CTAs per SM (query group 4)
constexpr int kStatusWords = 8;   // device status ints kept after the lengths in the arena
constexpr long long kWaitLimitCycles = 1ll << 31;  // ~1 s at 2 GHz: a staged-data wait gives up

// Orders of the 512 bytes of one plane (or of the sign words) of a 32-token tile. A token's 128
// bits are 16 bytes, byte k holding coordinates 8k..8k+7 (coordinate 8k + i in bit i).
//   kOrderByteLane: [16 byte-lanes][32 tokens] (values).
//   kOrderToken:    [32 tokens][16 B] (keys decoded on CUDA cores).
//   kOrderOctet:    bit-transposed for the tensor-core key contraction: [4 octets][32 words],
//                   octet o = tokens 8o..8o+7; word x = 8t + 2m + h, byte i of it covers
//                   coordinate 32m + 16h + 4t + i, bit j of that byte is token 8o + j.
constexpr int kOrderByteLane = 0;
constexpr int kOrderToken = 1;
constexpr int kOrderOctet = 2;

// Where one side (K or V) of an LM/SIGN1 cache keeps its fields inside a 32-token tile.
struct SideLayout {
  int bits = 0;         // code bit-planes
  int qjl = 0;          // 1 if a residual sign sketch is stored
  int order = 1;        // plane / sign-word order within a tile: one of the kOrder* below
  int m = 0;            // sketch rows
  int tile_bytes = 0;
  int off_planes = 0;   // [bits][512 B] (layout per order)
  int off_sketch = 0;   // [m/8 x 32 B] (layout per order)
  int off_norm = 0;     // [32] fp16
  int off_gamma = 0;    // [32] fp16
  float cent[8] = {};   // fp32 Lloyd-Max centroids (2^bits, ascending)
  float thr[7] = {};    // fp32 thresholds (2^bits - 1)
};

// FP4 latent cache tile: [32][latent/2] codes, [32][latent/16] E4M3 scales, [32][rope] bf16.
struct Fp4Layout {
  int latent = 0, rope = 0;
  int tile_bytes = 0;
  int off_codes = 0, off_scales = 0, off_rope = 0;
};

struct QuantizeParams {
  // LM/SIGN1: src[0] = K, src[1] = V, each [n_seq, heads, n_new, d].
  // FP4: src[0] = latent [n_seq, n_new, latent], src[1] = rope [n_seq, n_new, rope].
  const void* src[2];
  int bf16;
  int n_new, n_seq, heads;
  char* region[2];       // side region bases (FP4: region[0] only)
  int tiles_per_seq;
  const int* table;      // paged regions: block table [batch][pages_per_seq] (null: contiguous)
  int pages_per_seq, n_pages;
  SideLayout side[2];
  Fp4Layout fp4;
  const float* signs;    // [d] +-1 (per-head rotation: [heads][d])
  int signs_stride;      // 0: one diagonal for every head; d: head h reads signs + h * d
  const float* St;       // [d][m] transposed sketch matrix
  int* lens;             // device lengths, set to pos + n_new
  int skip_rotation;     // debug entry: src[0] already rotated and normalised (fp32)
  uint32_t* dbg_planes;  // debug outputs (skip_rotation only)
  uint32_t* dbg_sketch;
  uint16_t* dbg_gamma;
  int* err;              // cache status word: bit 0 set when a wait for staged data gave up
  long long wait_limit;  // SM clock cycles a block waits for staged data before giving up
  int seq[kMaxSeqPerLaunch];
  int pos[kMaxSeqPerLaunch];
  // Mixed-precision window caches. History appends (win_src): sequence s takes cnt[s] tokens, history
  // positions pos[s] ..; the token at sequence position sink + pos[s] + t comes from the bf16 ring
  // when it is below total0[s] (the length before the call), else from input row
  // (that position - total0[s]) of the call's src_rows rows. Window writes use total0 the same way.
  int win_src;
  // History appends whose tokens all come from the input (every sequence of the launch had the same
  // length, at most win_sink, before the call, and takes n_new = cnt[s] tokens): the tile kernel may
  // code them, history position pos[s] + t from input row src_row0 - total0[s] + t.
  int win_input_only, src_row0;
  const uint16_t* ring[2];  // bf16 window of K and V: [n_seq][heads][win_slots][d]
  int win_sink, win_recent, win_slots, src_rows;
  int win_kivi;             // KIVI caches: the window is the incomplete last key group (T % 128 tokens)
  char* kstats;             // KIVI caches: per (sequence, kv-head, 128-token group) fp16 key scales, zeros [2][d]
  int groups_per_seq;
  int total0[kMaxSeqPerLaunch];
  int cnt[kMaxSeqPerLaunch];
};

struct DecodeParams {
  const void* q;          // [B, Hq, d]
  int bf16;
  float* out;             // [B, Hq, d]
  float* pout;            // instead of out: merged softmax state [B, Hq, 2 + d] (m, l, unnormalised o)
  float* part;            // [B, Hq, splits, part_stride]
  int part_stride;        // 2 + d (+ m with a value sketch)
  int B, Hq, Hkv, group;
  int hsplit;             // tensor-core path: CTAs per (sequence, kv-head, split), G = group / hsplit heads each
  int splits, chunk;      // tokens per split (multiple of kTile)
  const int* lens;
  const char* kreg;
  const char* vreg;
  int tiles_per_seq;
  const int* table;       // paged regions: block table [B][pages_per_seq] (null: contiguous)
  int pages_per_seq, n_pages;
  SideLayout k, v;
  const float* signs;     // [d] (per-head rotation: [Hkv][d])
  int signs_stride;       // 0: one diagonal for every kv-head; d: kv-head hk reads signs + hk * d
  const float* S;         // [m][d]
  const float* St;        // [d][m]
  float logit_scale;      // softmax_scale * log2(e)
  unsigned char* qprep;   // per (sequence, kv-head) query digit tables (tensor-core path)
  int qprep_stride;       // bytes per (sequence, kv-head)
  int* err;               // cache status word: bit 0 set when a wait for staged data gave up
  long long wait_limit;   // SM clock cycles a kernel waits for staged data before giving up
  int debug_unset_wait;   // test entry: also wait once on a barrier nothing completes
  int cache_after_wait;   // fused step: the cache is written by this kernel's predecessor (wait first)
  int use_tc;             // decode on a tcgen05 kernel (one CTA per sequence, kv-head and split):
                          // 1 the lockstep kernel, 2 the warp-specialised one
  // mixed-precision window: bf16 K and V of the sink and recent tokens, [B][Hkv][win_slots][d] each;
  // lens above counts the coded history only, tot_lens every token; wpart [B][Hq][win_parts]
  // [part_stride] gets the softmax states of the window's parts of 64 slots, which the reduce merges
  // with the splits' (null: no window)
  const uint16_t* wk;
  const uint16_t* wv;
  int win_sink, win_recent, win_slots;
  const int* tot_lens;
  float* wpart;
  int win_parts;
  int win_fused;           // the mma.sync split kernel runs the window parts in CTAs past its splits'

  int win_kivi;            // KIVI caches: window = the incomplete last key group; outputs not rotated
  const char* kstats;      // KIVI caches: [B][Hkv][groups][2][d] fp16 key scales, zeros
  int groups_per_seq;
};

struct MlaParams {
  const void* q;          // [B, Hq, latent + rope]
  int bf16;
  float* out;             // [B, Hq, latent]
  float* pout;            // instead of out: merged softmax state [B, Hq, 2 + latent]
  float* part;            // [B, Hq, splits, 2 + latent]
  int B, Hq;
  int splits, chunk;
  const int* lens;
  const char* reg;
  int tiles_per_seq;
  Fp4Layout fp4;
  float logit_scale;      // softmax_scale * log2(e)
  int* err;               // cache status word (bit 0: a bounded wait gave up)
  long long wait_limit;   // SM clock cycles a kernel waits before giving up
};

// Reads cudaGetLastError() right after a kernel launch and, when it is cudaSuccess, adds one to
// the library's launch counter (kvq_kernel_launches).
cudaError_t launched();

// Launchers (kvq_quantize.cu, kvq_decode.cu, kvq_mla.cu). Return launched().
cudaError_t launch_quantize_lm(const QuantizeParams& p, int n_sides, cudaStream_t s);
cudaError_t launch_quantize_fp4(const QuantizeParams& p, cudaStream_t s);
// ev_mid (may be null) is recorded between the query prep and the split kernel (right before the
// split kernel when there is no prep).
// qp (may be null): a fused decode step's append, launched together with the query prep in one
// kernel (tensor-core path only; the caller checks mma_decode_supported).
cudaError_t launch_decode_lm(const DecodeParams& p, cudaStream_t s, cudaEvent_t ev_mid = nullptr,
                             const QuantizeParams* qp = nullptr);
bool mma_decode_supported(const DecodeParams& p);
// Resident CTAs per SM of the tensor-core decode kernel for a chunk of `chunk` tokens (shared
// memory and registers), as the split plan counts them.
int lm_mma_slots_per_sm(int group, const SideLayout& k, const SideLayout& v, int chunk, bool kivi = false);
// True when the tensor-core decode kernel handles this query group and code combination (the
// cache then stores its keys in kOrderOctet).
bool mma_modes_supported(int group, int k_bits, int k_qjl, int v_bits, int v_qjl);
int mma_prep_bytes(int k_bits, int k_qjl, int group);  // bytes of one (sequence, kv-head) prep area
cudaError_t launch_decode_lm_mma(const DecodeParams& p, cudaStream_t s, cudaEvent_t ev_mid, const QuantizeParams* qp);
cudaError_t launch_reduce_lm(const DecodeParams& p, cudaStream_t s);
// Query prep of the tensor-core paths in pieces of group / hsplit heads (or, with qp, the fused
// step's front kernel: append + query prep), as one launch.
cudaError_t launch_lm_query_prep(const DecodeParams& p, cudaStream_t s, const QuantizeParams* qp);
// The tcgen05 decode kernel (kvq_decode_tc.cu): one CTA per (sequence, kv-head, split) with all
// query heads of the group. tc_supported: this group and code combination have an instance.
bool tc_modes_supported(int group, int k_bits, int k_qjl, int v_bits, int v_qjl);
bool tc_decode_supported(const DecodeParams& p);
int tc_chunk_max(int group);     // largest chunk (tokens) of one CTA
cudaError_t launch_decode_lm_tc(const DecodeParams& p, cudaStream_t s, cudaEvent_t ev_mid, const QuantizeParams* qp);
// Warp-specialised tcgen05 kernel (kvq_decode_ws.cu): same modes, chunks and prep area as the tcgen05 kernel.
cudaError_t launch_decode_lm_ws(const DecodeParams& p, cudaStream_t s, cudaEvent_t ev_mid, const QuantizeParams* qp);
// The tcgen05 kernel's KIVI instance (chunks of whole 128-token key groups).
cudaError_t launch_decode_kivi_tc(const DecodeParams& p, cudaStream_t s);
// KIVI instance of the mma.sync split kernel (chunks of whole 128-token key groups).
cudaError_t launch_decode_kivi_mma(const DecodeParams& p, cudaStream_t s);
cudaError_t launch_decode_mla(const MlaParams& p, cudaStream_t s);
cudaError_t launch_reduce_mla(const MlaParams& p, cudaStream_t s);
bool mla_mma_supported(const MlaParams& p);
bool mla_umma_supported(const MlaParams& p);
// Log-sum-exp merge of n_parts softmax states [n_parts][rows][2 + dv] into out [rows][dv] (kvq_combine.cu).
// Mixed-precision window (kvq_window.cu): bf16 writes of appended tokens that stay in the window,
// and the window's softmax state for decode.
cudaError_t launch_window_write(const QuantizeParams& p, cudaStream_t s);
// KIVI caches (kvq_kivi.cu): code every 128-token group an append completes (tail and input rows).
cudaError_t launch_kivi_groups(const QuantizeParams& p, int max_groups, cudaStream_t s);
cudaError_t launch_decode_kivi(const DecodeParams& p, cudaStream_t s);
cudaError_t launch_window_decode(const DecodeParams& p, cudaStream_t s);
cudaError_t launch_combine_partials(const float* parts, int n_parts, int rows, int dv, float* out, cudaStream_t s);
cudaError_t launch_decode_mla_umma(const MlaParams& p, cudaStream_t s);
cudaError_t launch_decode_mla_mma(const MlaParams& p, cudaStream_t s);

// Host Lloyd-Max tables (lloyd_max.cpp): fp64 fixed-point iteration rounded to fp32.
void lloyd_max_f32(int bits, float* centroids, float* thresholds);

}  // namespace kvq

// Host object behind the opaque kvq_cache handle.
struct kvq_cache {
  kvq_cfg cfg;
  int batch = 0, capacity = 0, tiles_per_seq = 0, sms = 148;
  int signs_stride = 0;     // 0, or kHeadDim when every kv-head has its own rotation diagonal
  int device = -1;          // the CUDA device whose memory holds the arena (current at init)
  bool tc = false;          // LM decode runs on a tcgen05 kernel (else mma.sync / CUDA cores)
  bool ws = false;          // ... the warp-specialised one
  int sink = 0, recent = 0; // mixed-precision window (0, 0: none)
  const int* table = nullptr;  // paged caches: caller's device block table [batch][pages_per_seq]
  int pages_per_seq = 0, n_pages = 0;
  int* d_hlens = nullptr;   // window caches: coded history length per sequence (the decode kernels' lens)
  uint16_t* d_win = nullptr;// window caches: bf16 K then V window, [batch][kv-heads][sink + recent][d] each
  std::vector<int> hlens;   // host mirror of d_hlens
  bool kivi = false;        // KIVI codes (no rotation); the window is the incomplete last key group
  bool kivi_tc = false;     // KIVI decode on the tcgen05 kernel
  bool kivi_cuda = false;   // KIVI decode on the CUDA-core kernel (neither: the mma.sync kernel)
  char* d_kstats = nullptr; // KIVI: [batch][kv-heads][groups][2][d] fp16 key scales and zeros
  int groups_per_seq = 0;
  char* dev = nullptr;
  size_t dev_bytes = 0;
  int* d_lens = nullptr;
  int* d_status = nullptr;  // kStatusWords device ints after the lengths (zeroed at init)
  float* d_signs = nullptr;
  float* d_S = nullptr;
  float* d_St = nullptr;
  char* d_k = nullptr;
  char* d_v = nullptr;
  size_t k_region = 0, v_region = 0;
  kvq::SideLayout k, v;
  kvq::Fp4Layout fp4;
  bool is_fp4 = false;
  std::vector<int> lens;
  std::vector<float> h_tables;  // staging for the asynchronous table copies
};
