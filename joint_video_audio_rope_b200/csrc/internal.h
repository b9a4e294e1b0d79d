// Launchers shared between the C-ABI front end (mmdit_api.cu) and the kernel
// translation units.  Host-only declarations; not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <nvtx3/nvToolsExt.h>

#include <atomic>
#include <mutex>

#include "common.cuh"

namespace mmdit {

// NVTX range around one C-ABI call (named after the call), so that a
// profiler timeline shows which library call launched which kernels.  The
// NVTX header is a no-op unless a tool injects itself.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};
#define MMDIT_NVTX(name) ::mmdit::NvtxRange mmdit_nvtx_range_(name)

constexpr int kMaxDevices = 64;  // device indices the per-device state covers
constexpr int kMaxBlocks = 6000; // key/query blocks of one block-sparse problem

// Runs fn() (returning cudaError_t) once per device index for each call site
// (each lambda type has its own state), thread-safe; a failed fn() is retried
// on the next call.  Used for per-device function attributes.
template <typename F>
cudaError_t once_per_device(int dev, F fn) {
  static std::atomic<bool> done[kMaxDevices] = {};
  static std::mutex mu;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  std::lock_guard<std::mutex> lock(mu);
  if (done[dev].load(std::memory_order_relaxed)) return cudaSuccess;
  const cudaError_t e = fn();
  if (e == cudaSuccess) done[dev].store(true, std::memory_order_release);
  return e;
}

// RoPE (rope.cu)
cudaError_t launch_rope(void* q, void* k, const mmdit_tensor_desc& d, const DevLayout& L,
                        const RopeTab& tab, cudaStream_t s);

// fp32 SIMT attention (attn_f32.cu): o = softmax(q k^T scale) v per (b, h);
// optional lse [B, H, Nq].
struct F32AttnArgs {
  const float *q, *k, *v;
  float* o;
  float* lse;
  int B, H, D, Nq, Nkv;
  long long q_st, q_sb, k_st, k_sb, v_st, v_sb, o_st, o_sb;  // strides in elements
  float scale;
};
cudaError_t launch_attn_f32(const F32AttnArgs& a, cudaStream_t s);

// tcgen05 bf16 attention (attn_tc.cu); the dense or block-sparse mode is a
// template parameter of the kernel, chosen by whether `order` is set

struct AttnProblem {
  CUtensorMap tmQ, tmK, tmV;  // 4D maps {channel, head, token, batch}, box {64,1,64,1}
  CUtensorMap tmO;            // bf16 output (dense mode), box {32 or 64,1,32,1}
  __nv_bfloat16* o;           // output (dense/sparse), or nullptr when writing partials
  long long o_st, o_sb;       // output strides (elements)
  float* lse;                 // [B, H, Nq] or nullptr
  float* part_o;              // split-KV partials [split][B][H][Nq_pad][128] (unnormalised)
  float* part_ml;             // split-KV partials [split][B][H][Nq_pad][2] (m*log2e*scale, l)
  int Nq, Nkv, H, B;
  int n_qtiles;               // ceil(Nq / 256) (dense) or number of groups (sparse)
  int n_splits;               // KV splits per (q tile pair, head, batch)
  int kv_per_split;           // tokens per split, multiple of 128
  int ctas;                   // work items: n_qtiles * H * B * n_splits
  // sparse mode: the query groups and the merged key lists (n_qtiles = the
  // groups' capacity per batch item), the block table, and the list of the
  // work items that exist (ids (b H + h) n_qtiles + g, in index order)
  const int4* groups;         // [B][n_qtiles]: {first block, n blocks, start token, n tokens}
  const int* n_groups;        // [B]
  const uint4* ulist;         // [B][H][n_qtiles][ucap]: {start, len, seg masks 0|1, seg masks 2|3}
  const int* ucnt;            // [B][H][n_qtiles]
  int ucap;
  const int2* tab;            // [B][tab_cap] {start, length} of every block
  int tab_cap;
  const int* order;           // [*n_order] item ids; nullptr: items in index order
  const int* n_order;
  int rope_q;                 // rotate Q tiles in shared memory after loading
  const int* q_count;         // dense mode, optional: valid query rows per batch item
                              // (device; rows from q_count[b] on are not computed)
  float* row_sq;              // dense mode, optional: [B][Nq][H] squared L2 norm of every
                              // normalised output row (fp32, before the bf16 rounding)
};

// One attention problem per launch: every field of `prob` sits at a fixed
// offset of the kernel's parameter block, so the kernel reads it with
// immediate constant-bank operands instead of indexed loads.
struct AttnParams {
  AttnProblem prob;
  int q_tiles;                // 128-row Q tiles per CTA: 2 (default) or 1
  int persistent;             // 0: one CTA per work item; 1: one CTA per SM slot, looping
  float scale_log2;           // softmax scale * log2(e)
  DevLayout layout;           // for fused Q RoPE
  RopeTab rope;
  int* err;                   // device error flag
};

cudaError_t launch_attn_tc(const AttnParams& p, cudaStream_t s);
// Queries over at most kShortKeys keys (attn_short.cu): every key in one
// N = 256 tile, single-pass softmax, K/V resident per (batch, head).  Uses the
// fields of a dense persistent one-tile problem (tmQ, tmK, tmV, tmO with a
// 32-channel store box, Nq, Nkv, H, B, row_sq).
constexpr int kShortKeys = 256;
cudaError_t launch_attn_short(const AttnParams& p, cudaStream_t s);
// Both directions of the audio<->video cross-attention on one stream: audio
// queries over the video keys (split-KV partials into part_o / part_ml), video
// queries over the audio keys, then the merge of the partials.
// With row_sq and video_norm non-NULL, the video-query launch also writes the
// squared norm of every (token, head) output row into row_sq [B][Nv][H] and
// video_norm [B][Nv] receives the L2 norm of each video token's output over
// all heads (launch_cross_norms).
int launch_cross(const void* qv, const void* kv, const void* vv, const void* qa, const void* ka,
                 const void* va, void* o_video, void* o_audio, const mmdit_tensor_desc& video,
                 const mmdit_tensor_desc& audio, float scale, int splits, int kv_per_split,
                 float* part_o, float* part_ml, cudaStream_t s, float* row_sq = nullptr,
                 float* video_norm = nullptr);
cudaError_t launch_cross_norms(const float* sq, int heads, long long n_rows, float* a,
                               cudaStream_t s);
// Split of the video keys for the audio-query direction of the cross
// attention (mmdit_api.cu): audio query tiles of 256 rows, `splits` key ranges
// of kv_per_split tokens (a multiple of 128), and the partial-result sizes.
struct CrossPlan {
  int n_qtiles_a, splits, kv_per_split, nq_pad;
  size_t part_o_bytes, part_ml_bytes;
};
CrossPlan plan_cross(const mmdit_tensor_desc* video, const mmdit_tensor_desc* audio);
int attn_rows_per_cta(int q_tiles);  // query rows one CTA covers
int attn_store_cols(int q_tiles);    // channels per output store box
cudaError_t launch_split_combine(const float* part_o, const float* part_ml, __nv_bfloat16* o,
                                 long long o_st, long long o_sb, int n_splits, int B, int H,
                                 int Nq, int Nq_pad, cudaStream_t s);

// block-sparse attention: query blocks per CTA group are bounded by the rows
// of the kernel shape used (kSparseQTiles 128-row Q tiles) and 8 blocks per
// Q tile (membership masks are 16 bits wide)
constexpr int kSparseQTiles = 2;
constexpr int kGroupTokens = 128 * kSparseQTiles;
constexpr int kGroupBlocks = 8 * kSparseQTiles;
constexpr int kMaxBlockTokens = 256;  // longest block of any block table

// block selection and the sparse-attention preparation (select.cu).  Block
// tables: per batch item `maxb` int2 {start token, length} in storage order
// and a block count; pooled means [B][H][maxb][128]; scores [B][H][maxb][ld].
cudaError_t launch_grid_table(int T, int H, int W, int nblk, int B, int maxb, int2* tab,
                              int* tab_n, cudaStream_t s);
size_t select_scores_ld(int maxb);
cudaError_t launch_pool(const __nv_bfloat16* q, const __nv_bfloat16* k, const mmdit_tensor_desc& d,
                        const int2* tab, const int* tab_n, int maxb, float* qbar, float* kbar,
                        int* err, cudaStream_t s);
cudaError_t launch_select(const float* qbar, const float* kbar, const int* tab_n, int B, int H,
                          int maxb, int top_k, float top_p, float scale, int cap, float* S,
                          int32_t* idx, int32_t* cnt, int* err, cudaStream_t s);
cudaError_t launch_groups(const int2* tab, const int* tab_n, int B, int maxb, int N, int maxg,
                          int4* groups, int* n_groups, int* err, cudaStream_t s);
cudaError_t launch_union(const int32_t* idx, const int32_t* cnt, int cap, const int2* tab,
                         const int* tab_n, int maxb, int N, const int4* groups,
                         const int* n_groups, int maxg, int B, int H, int ucap, uint4* ulist,
                         int* ucnt, int* err, cudaStream_t s);
cudaError_t launch_schedule(const int* n_groups, int maxg, int B, int H, int* order,
                            int* n_order, cudaStream_t s);

// helpers (mmdit_api.cu)
int* device_error_flag();  // device address of this device's error word
int fail(int code, const char* fmt, ...);  // sets the thread-local message
int cuda_fail(cudaError_t e, const char* what);
bool aligned16(const void* p);
int check_desc(const mmdit_tensor_desc* d, const char* name);
int check_layout(const mmdit_layout* L, int n_tokens);  // segments sum to n_tokens, valid kinds
int make_map(CUtensorMap* m, const void* base, const mmdit_tensor_desc& d, int n_tokens,
             const char* name);
// Store map of a bf16 [B, N, heads, 128] output with the strides of `d`: box
// {cols channels, 1 head, 32 tokens, 1}, cols = 32 or 64 with the 64- or
// 128-byte swizzle (the attention epilogue's staging layout).
int make_store_map(CUtensorMap* m, void* base, const mmdit_tensor_desc& d, int n_tokens,
                   int cols, const char* name);
int check_sm100();
size_t align256(size_t x);

}  // namespace mmdit
