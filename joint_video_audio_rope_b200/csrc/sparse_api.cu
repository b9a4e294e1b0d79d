// C-ABI entry points of the block-sparse mode (declared in include/mmdit.h):
// hybrid top-k / top-p block selection and attention restricted to the
// selected blocks (Prism guide, arXiv 2610.05416, Method section 3), over
// either the fixed 4x4x4 blocks of a block-major video segment or any block
// table -- in particular the content-adaptive blocks of mmdit_adaptive_plan
// (Method sections 1-2).  Both forms run the same kernels (select.cu and the
// sparse mode of attn_tc.cu): the 4x4x4 form first writes the grid's block
// table into its workspace.  Arguments are validated before any launch.
#include "internal.h"

namespace mmdit {

namespace {

// single BLOCK444 video segment -> grid and block count
int sparse_layout(const mmdit_layout* L, const mmdit_tensor_desc* d, int& T, int& H, int& W,
                  int& nblk) {
  int rc = check_layout(L, d->n_tokens);
  if (rc) return rc;
  if (L->n_seg != 1 || L->seg[0].kind != MMDIT_SEG_VIDEO || L->seg[0].order != MMDIT_ORDER_BLOCK444)
    return fail(MMDIT_EINVAL, "block-sparse calls need exactly one BLOCK444 video segment");
  T = L->seg[0].T;
  H = L->seg[0].H;
  W = L->seg[0].W;
  const long long nb = (long long)((T + 3) / 4) * ((H + 3) / 4) * ((W + 3) / 4);
  if (nb > kMaxBlocks)
    return fail(MMDIT_EUNSUPPORTED, "%lld blocks; at most %d are supported", nb, kMaxBlocks);
  nblk = (int)nb;
  return MMDIT_OK;
}

int host_block_len(int T, int H, int W, int b) {
  const int nhb = (H + 3) / 4, nwb = (W + 3) / 4;
  const int tb = b / (nhb * nwb), r = b % (nhb * nwb), hb = r / nwb, wb = r % nwb;
  return std::min(4, T - 4 * tb) * std::min(4, H - 4 * hb) * std::min(4, W - 4 * wb);
}

// greedy grouping of query blocks (<= kGroupTokens tokens, <= kGroupBlocks
// blocks); the device groups_kernel applies the same rule and writes the table.
int host_group_count(int T, int H, int W, int nblk) {
  int g = 0, nb = 0, tokens = 0;
  for (int b = 0; b < nblk; ++b) {
    const int len = host_block_len(T, H, W, b);
    if (nb == kGroupBlocks || tokens + len > kGroupTokens) {
      ++g;
      nb = 0;
      tokens = 0;
    }
    ++nb;
    tokens += len;
  }
  return g + (nb > 0 ? 1 : 0);
}

// Bounds of a block table of `maxb` entries over N tokens per batch item:
// query groups and merged-list entries per group.  The greedy grouping closes
// a group either at kGroupBlocks blocks or when the next block would pass
// kGroupTokens tokens, so two consecutive groups of the second kind hold more
// than kGroupTokens tokens together: groups <= maxb / 16 + N / 128 + 1.  A
// block of L tokens gives at most ceil(L / 64) <= L / 64 + 1 entries.
int table_group_bound(int maxb, int N) {
  const long long g = (maxb + kGroupBlocks - 1) / kGroupBlocks + (N + kGroupTokens / 2 - 1) /
                                                                     (kGroupTokens / 2) + 1;
  return (int)std::min<long long>(maxb, g);
}
int table_entry_bound(int maxb, int N) { return (N + 63) / 64 + maxb; }

// Workspace of the selection: pooled means, scores (and the grid's table).
struct SelectWs {
  size_t tab, tab_n, qbar, kbar, scores, bytes;
};
SelectWs select_ws(int B, int H, int maxb, bool with_table) {
  SelectWs w{};
  size_t off = 0;
  auto take = [&](size_t n) {
    const size_t o = off;
    off += align256(n);
    return o;
  };
  w.tab = with_table ? take(sizeof(int2) * (size_t)B * maxb) : 0;
  w.tab_n = with_table ? take(sizeof(int) * (size_t)B) : 0;
  w.qbar = take(sizeof(float) * (size_t)B * H * maxb * 128);
  w.kbar = take(sizeof(float) * (size_t)B * H * maxb * 128);
  w.scores = take(sizeof(float) * (size_t)B * H * maxb * select_scores_ld(maxb));
  w.bytes = off;
  return w;
}

// Workspace of the sparse attention: groups, merged lists, item order (and
// the grid's table).
struct SparseWs {
  size_t tab, tab_n, groups, n_groups, ulist, ucnt, order, n_order, bytes;
  int maxg, ucap;
};
SparseWs sparse_ws(int B, int H, int maxb, int maxg, int ucap, bool with_table) {
  SparseWs w{};
  size_t off = 0;
  auto take = [&](size_t n) {
    const size_t o = off;
    off += align256(n);
    return o;
  };
  w.maxg = maxg;
  w.ucap = ucap;
  w.tab = with_table ? take(sizeof(int2) * (size_t)B * maxb) : 0;
  w.tab_n = with_table ? take(sizeof(int) * (size_t)B) : 0;
  w.groups = take(sizeof(int4) * (size_t)B * maxg);
  w.n_groups = take(sizeof(int) * (size_t)B);
  w.ulist = take(sizeof(uint4) * (size_t)B * H * maxg * ucap);
  w.ucnt = take(sizeof(int) * (size_t)B * H * maxg);
  w.order = take(sizeof(int) * (size_t)B * H * maxg);
  w.n_order = take(sizeof(int));
  w.bytes = off;
  return w;
}

int check_workspace(void* ws, size_t bytes, size_t need, const char* name) {
  if (ws == nullptr || bytes < need)
    return fail(MMDIT_EWORKSPACE, "%s: workspace needs %zu bytes", name, need);
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
    return fail(MMDIT_EINVAL, "%s: workspace must be 256-byte aligned", name);
  return MMDIT_OK;
}

int check_select_args(const void* q, const void* k, const mmdit_tensor_desc* desc, int top_k,
                      float top_p, float scale, int32_t* idx, int32_t* cnt, const char* name) {
  int rc = check_desc(desc, name);
  if (rc) return rc;
  if (desc->dtype != MMDIT_BF16) return fail(MMDIT_EUNSUPPORTED, "%s: bf16 only", name);
  if (!q || !k || !idx || !cnt)
    return fail(MMDIT_EINVAL, "%s: q, k, block_idx, block_cnt must be non-NULL", name);
  if (!aligned16(q) || !aligned16(k)) return fail(MMDIT_EINVAL, "%s: 16-byte alignment", name);
  if (top_k < 0) return fail(MMDIT_EINVAL, "%s: top_k < 0", name);
  if (!(top_p >= 0.f && top_p <= 1.f)) return fail(MMDIT_EINVAL, "%s: top_p outside [0, 1]", name);
  if (!(scale > 0.f) || !isfinite(scale)) return fail(MMDIT_EINVAL, "%s: scale must be > 0", name);
  return MMDIT_OK;
}

int check_sparse_args(const void* q, const void* k, const void* v, const void* o,
                      const mmdit_tensor_desc* desc, const int32_t* idx, const int32_t* cnt,
                      float scale, const char* name) {
  int rc = check_desc(desc, name);
  if (rc) return rc;
  if (desc->dtype != MMDIT_BF16) return fail(MMDIT_EUNSUPPORTED, "%s: bf16 only", name);
  if (!q || !k || !v || !o || !idx || !cnt)
    return fail(MMDIT_EINVAL, "%s: every pointer must be non-NULL", name);
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return fail(MMDIT_EINVAL, "%s: 16-byte alignment", name);
  if (o == q || o == k || o == v) return fail(MMDIT_EINVAL, "%s: o aliases an input", name);
  if (!(scale > 0.f) || !isfinite(scale)) return fail(MMDIT_EINVAL, "%s: scale must be > 0", name);
  return MMDIT_OK;
}

int run_select(const void* q, const void* k, const mmdit_tensor_desc& d, const int2* tab,
               const int* tab_n, int maxb, const SelectWs& w, char* ws, int top_k, float top_p,
               float scale, int cap, int32_t* idx, int32_t* cnt, int* err, cudaStream_t s) {
  float* qbar = reinterpret_cast<float*>(ws + w.qbar);
  float* kbar = reinterpret_cast<float*>(ws + w.kbar);
  float* S = reinterpret_cast<float*>(ws + w.scores);
  cudaError_t e = launch_pool((const __nv_bfloat16*)q, (const __nv_bfloat16*)k, d, tab, tab_n,
                              maxb, qbar, kbar, err, s);
  if (e == cudaSuccess)
    e = launch_select(qbar, kbar, tab_n, d.batch, d.heads, maxb, top_k, top_p, scale, cap, S, idx,
                      cnt, err, s);
  return e == cudaSuccess ? MMDIT_OK : cuda_fail(e, "block_select launch");
}

int run_sparse(const void* q, const void* k, const void* v, void* o, const mmdit_tensor_desc& d,
               const int2* tab, const int* tab_n, int maxb, const SparseWs& w, char* ws,
               const int32_t* idx, const int32_t* cnt, int cap, float scale, int* err,
               cudaStream_t s) {
  int4* groups = reinterpret_cast<int4*>(ws + w.groups);
  int* n_groups = reinterpret_cast<int*>(ws + w.n_groups);
  uint4* ulist = reinterpret_cast<uint4*>(ws + w.ulist);
  int* ucnt = reinterpret_cast<int*>(ws + w.ucnt);
  int* order = reinterpret_cast<int*>(ws + w.order);
  int* n_order = reinterpret_cast<int*>(ws + w.n_order);
  cudaError_t e = launch_groups(tab, tab_n, d.batch, maxb, d.n_tokens, w.maxg, groups, n_groups,
                                err, s);
  if (e == cudaSuccess)
    e = launch_union(idx, cnt, cap, tab, tab_n, maxb, d.n_tokens, groups, n_groups, w.maxg,
                     d.batch, d.heads, w.ucap, ulist, ucnt, err, s);
  if (e == cudaSuccess)
    e = launch_schedule(n_groups, w.maxg, d.batch, d.heads, order, n_order, s);
  if (e != cudaSuccess) return cuda_fail(e, "sparse_attn prep launch");
  int rc;
  AttnParams p{};
  AttnProblem& pr = p.prob;
  if ((rc = make_map(&pr.tmQ, q, d, d.n_tokens, "q")) ||
      (rc = make_map(&pr.tmK, k, d, d.n_tokens, "k")) ||
      (rc = make_map(&pr.tmV, v, d, d.n_tokens, "v")))
    return rc;
  pr.o = (__nv_bfloat16*)o;
  pr.o_st = d.stride_tok;
  pr.o_sb = d.stride_batch;
  pr.Nq = pr.Nkv = d.n_tokens;
  pr.H = d.heads;
  pr.B = d.batch;
  pr.n_qtiles = w.maxg;
  pr.n_splits = 1;
  pr.kv_per_split = 0;
  pr.ctas = w.maxg * pr.H * pr.B;
  pr.groups = groups;
  pr.n_groups = n_groups;
  pr.ulist = ulist;
  pr.ucnt = ucnt;
  pr.ucap = w.ucap;
  pr.tab = tab;
  pr.tab_cap = maxb;
  pr.order = order;
  pr.n_order = n_order;
  p.q_tiles = kSparseQTiles;
  p.persistent = 0;  // one CTA per listed item: the hardware balances the ragged lists
  p.scale_log2 = scale * 1.4426950408889634f;
  p.err = err;
  e = launch_attn_tc(p, s);
  return e == cudaSuccess ? MMDIT_OK : cuda_fail(e, "sparse attn launch");
}

// block table argument checks (the table itself lives on the device)
int check_table_args(const mmdit_tensor_desc* desc, const int32_t* blocks, const int32_t* n_blocks,
                     int max_blocks, const char* name) {
  if (!blocks || !n_blocks) return fail(MMDIT_EINVAL, "%s: blocks and n_blocks must be non-NULL", name);
  if ((reinterpret_cast<uintptr_t>(blocks) & 7u) != 0)
    return fail(MMDIT_EINVAL, "%s: blocks must be 8-byte aligned", name);
  if (max_blocks < 1 || max_blocks > kMaxBlocks)
    return fail(MMDIT_EINVAL, "%s: max_blocks %d outside [1, %d]", name, max_blocks, kMaxBlocks);
  (void)desc;
  return MMDIT_OK;
}

}  // namespace

}  // namespace mmdit

using namespace mmdit;

extern "C" {

int mmdit_num_blocks(const mmdit_layout* L) {
  if (L == nullptr || L->n_seg != 1 || L->seg[0].kind != MMDIT_SEG_VIDEO ||
      L->seg[0].order != MMDIT_ORDER_BLOCK444 || L->seg[0].T < 1 || L->seg[0].H < 1 ||
      L->seg[0].W < 1)
    return 0;
  return ((L->seg[0].T + 3) / 4) * ((L->seg[0].H + 3) / 4) * ((L->seg[0].W + 3) / 4);
}

size_t mmdit_block_select_workspace_size(const mmdit_tensor_desc* desc, const mmdit_layout* layout) {
  int T, H, W, nblk;
  if (check_desc(desc, "block_select") || sparse_layout(layout, desc, T, H, W, nblk)) return 0;
  return select_ws(desc->batch, desc->heads, nblk, true).bytes;
}

int mmdit_block_select(const void* q, const void* k, const mmdit_tensor_desc* desc,
                       const mmdit_layout* layout, int top_k, float top_p, float scale, int cap,
                       int32_t* block_idx, int32_t* block_cnt, void* workspace, size_t ws_bytes,
                       mmdit_stream_t stream) {
  MMDIT_NVTX("mmdit_block_select");
  int rc = check_select_args(q, k, desc, top_k, top_p, scale, block_idx, block_cnt, "block_select");
  if (rc) return rc;
  int T, H, W, nblk;
  if ((rc = sparse_layout(layout, desc, T, H, W, nblk))) return rc;
  if (cap < nblk) return fail(MMDIT_EINVAL, "block_select: cap %d < number of blocks %d", cap, nblk);
  const SelectWs w = select_ws(desc->batch, desc->heads, nblk, true);
  if ((rc = check_workspace(workspace, ws_bytes, w.bytes, "block_select"))) return rc;
  if ((rc = check_sm100())) return rc;
  int* err = device_error_flag();
  if (err == nullptr) return fail(MMDIT_ECUDA, "device error flag unavailable");
  char* ws = static_cast<char*>(workspace);
  int2* tab = reinterpret_cast<int2*>(ws + w.tab);
  int* tab_n = reinterpret_cast<int*>(ws + w.tab_n);
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = launch_grid_table(T, H, W, nblk, desc->batch, nblk, tab, tab_n, s);
  if (e != cudaSuccess) return cuda_fail(e, "block_select table launch");
  return run_select(q, k, *desc, tab, tab_n, nblk, w, ws, top_k, top_p, scale, cap, block_idx,
                    block_cnt, err, s);
}

size_t mmdit_sparse_attn_workspace_size(const mmdit_tensor_desc* desc, const mmdit_layout* layout,
                                        int) {
  int T, H, W, nblk;
  if (check_desc(desc, "sparse_attn") || sparse_layout(layout, desc, T, H, W, nblk)) return 0;
  return sparse_ws(desc->batch, desc->heads, nblk, host_group_count(T, H, W, nblk), nblk, true)
      .bytes;
}

int mmdit_sparse_attn(const void* q, const void* k, const void* v, void* o,
                      const mmdit_tensor_desc* desc, const mmdit_layout* layout,
                      const int32_t* block_idx, const int32_t* block_cnt, int cap, float scale,
                      void* workspace, size_t ws_bytes, mmdit_stream_t stream) {
  MMDIT_NVTX("mmdit_sparse_attn");
  int rc = check_sparse_args(q, k, v, o, desc, block_idx, block_cnt, scale, "sparse_attn");
  if (rc) return rc;
  int T, H, W, nblk;
  if ((rc = sparse_layout(layout, desc, T, H, W, nblk))) return rc;
  if (cap < nblk) return fail(MMDIT_EINVAL, "sparse_attn: cap %d < number of blocks %d", cap, nblk);
  // 4x4x4 blocks hold <= 64 tokens: one list entry per block at most
  const SparseWs w = sparse_ws(desc->batch, desc->heads, nblk, host_group_count(T, H, W, nblk),
                               nblk, true);
  if ((rc = check_workspace(workspace, ws_bytes, w.bytes, "sparse_attn"))) return rc;
  if ((rc = check_sm100())) return rc;
  int* err = device_error_flag();
  if (err == nullptr) return fail(MMDIT_ECUDA, "device error flag unavailable");
  char* ws = static_cast<char*>(workspace);
  int2* tab = reinterpret_cast<int2*>(ws + w.tab);
  int* tab_n = reinterpret_cast<int*>(ws + w.tab_n);
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = launch_grid_table(T, H, W, nblk, desc->batch, nblk, tab, tab_n, s);
  if (e != cudaSuccess) return cuda_fail(e, "sparse_attn table launch");
  return run_sparse(q, k, v, o, *desc, tab, tab_n, nblk, w, ws, block_idx, block_cnt, cap, scale,
                    err, s);
}

size_t mmdit_block_select_table_workspace_size(const mmdit_tensor_desc* desc, int max_blocks) {
  if (check_desc(desc, "block_select_table") || max_blocks < 1 || max_blocks > kMaxBlocks) return 0;
  return select_ws(desc->batch, desc->heads, max_blocks, false).bytes;
}

int mmdit_block_select_table(const void* q, const void* k, const mmdit_tensor_desc* desc,
                             const int32_t* blocks, const int32_t* n_blocks, int max_blocks,
                             int top_k, float top_p, float scale, int cap, int32_t* block_idx,
                             int32_t* block_cnt, void* workspace, size_t ws_bytes,
                             mmdit_stream_t stream) {
  MMDIT_NVTX("mmdit_block_select_table");
  int rc = check_select_args(q, k, desc, top_k, top_p, scale, block_idx, block_cnt,
                             "block_select_table");
  if (rc) return rc;
  if ((rc = check_table_args(desc, blocks, n_blocks, max_blocks, "block_select_table"))) return rc;
  if (cap < max_blocks)
    return fail(MMDIT_EINVAL, "block_select_table: cap %d < max_blocks %d", cap, max_blocks);
  const SelectWs w = select_ws(desc->batch, desc->heads, max_blocks, false);
  if ((rc = check_workspace(workspace, ws_bytes, w.bytes, "block_select_table"))) return rc;
  if (desc->n_tokens == 0) return MMDIT_OK;
  if ((rc = check_sm100())) return rc;
  int* err = device_error_flag();
  if (err == nullptr) return fail(MMDIT_ECUDA, "device error flag unavailable");
  return run_select(q, k, *desc, reinterpret_cast<const int2*>(blocks), n_blocks, max_blocks, w,
                    static_cast<char*>(workspace), top_k, top_p, scale, cap, block_idx,
                    block_cnt, err, (cudaStream_t)stream);
}

size_t mmdit_sparse_attn_table_workspace_size(const mmdit_tensor_desc* desc, int max_blocks) {
  if (check_desc(desc, "sparse_attn_table") || max_blocks < 1 || max_blocks > kMaxBlocks) return 0;
  return sparse_ws(desc->batch, desc->heads, max_blocks,
                   table_group_bound(max_blocks, desc->n_tokens),
                   table_entry_bound(max_blocks, desc->n_tokens), false)
      .bytes;
}

int mmdit_sparse_attn_table(const void* q, const void* k, const void* v, void* o,
                            const mmdit_tensor_desc* desc, const int32_t* blocks,
                            const int32_t* n_blocks, int max_blocks, const int32_t* block_idx,
                            const int32_t* block_cnt, int cap, float scale, void* workspace,
                            size_t ws_bytes, mmdit_stream_t stream) {
  MMDIT_NVTX("mmdit_sparse_attn_table");
  int rc = check_sparse_args(q, k, v, o, desc, block_idx, block_cnt, scale, "sparse_attn_table");
  if (rc) return rc;
  if ((rc = check_table_args(desc, blocks, n_blocks, max_blocks, "sparse_attn_table"))) return rc;
  if (cap < max_blocks)
    return fail(MMDIT_EINVAL, "sparse_attn_table: cap %d < max_blocks %d", cap, max_blocks);
  const SparseWs w = sparse_ws(desc->batch, desc->heads, max_blocks,
                               table_group_bound(max_blocks, desc->n_tokens),
                               table_entry_bound(max_blocks, desc->n_tokens), false);
  if ((rc = check_workspace(workspace, ws_bytes, w.bytes, "sparse_attn_table"))) return rc;
  if (desc->n_tokens == 0) return MMDIT_OK;
  if ((rc = check_sm100())) return rc;
  int* err = device_error_flag();
  if (err == nullptr) return fail(MMDIT_ECUDA, "device error flag unavailable");
  return run_sparse(q, k, v, o, *desc, reinterpret_cast<const int2*>(blocks), n_blocks,
                    max_blocks, w, static_cast<char*>(workspace), block_idx, block_cnt, cap,
                    scale, err, (cudaStream_t)stream);
}

}  // extern "C"
