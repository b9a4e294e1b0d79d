// Mask-guided region-restricted attention: the conditional refinement of the
// Refiner, which with a spatial mask refines only the target region (blog
// section 4.2).  For every video token whose mask value is non-zero, its row
// of O = softmax(Q K^T * scale) V over all tokens of its batch item is
// computed; every other row of O is left untouched.
//
// Path (all on the caller's stream, scratch in the caller's workspace):
//   1. mask_rows_kernel   -- per batch item, the sequence index of every
//                            masked video token (arbitrary order) and their
//                            count;
//   2. move_rows_kernel<true>  -- those Q rows into a compact [B, Nv, H, 128]
//                            buffer (gather);
//   3. attn_tc_kernel     -- dense attention of the compact rows over every
//                            key, the per-batch count bounding the query rows
//                            (work items past it compute nothing);
//   4. move_rows_kernel<false> -- the compact O rows back to their tokens
//                            (scatter).
// Rows are independent in attention, so the order of the row list changes no
// value.  Nv (video tokens per batch item) sizes the scratch: the count is
// only known on the device, and nothing here waits for it on the host.
#include "internal.h"

namespace mmdit {

namespace {

// Video segments of the layout, in sequence order, as the mask indexes them.
struct VideoRows {
  int n_seg;
  int ord0[MMDIT_MAX_SEGMENTS];    // first video ordinal of the segment
  int tok0[MMDIT_MAX_SEGMENTS];    // first token of the segment in the sequence
  int frame0[MMDIT_MAX_SEGMENTS];  // first mask frame of the segment
  int hw;                          // H * W, shared by every video segment
  int n_video;                     // video tokens per batch item
  int frames;                      // mask frames per batch item
};

// One thread per video token of batch item blockIdx.y: a token whose mask
// value is non-zero appends its sequence index to the item's row list (one
// atomic per warp).
__global__ void __launch_bounds__(256) mask_rows_kernel(const uint8_t* __restrict__ mask,
                                                        VideoRows vr, int* __restrict__ count,
                                                        int* __restrict__ rows) {
  const int b = blockIdx.y;
  const int i = blockIdx.x * 256 + threadIdx.x;
  bool on = false;
  int tok = 0;
  if (i < vr.n_video) {
    int s = 0;
    while (s + 1 < vr.n_seg && i >= vr.ord0[s + 1]) ++s;
    const int local = i - vr.ord0[s];
    const int f = vr.frame0[s] + local / vr.hw;
    on = mask[((long long)b * vr.frames + f) * vr.hw + local % vr.hw] != 0;
    tok = vr.tok0[s] + local;
  }
  const unsigned ballot = __ballot_sync(0xffffffffu, on);
  if (ballot == 0u) return;  // the same for every lane of the warp
  const int lane = threadIdx.x & 31;
  const int leader = __ffs(ballot) - 1;
  int base = 0;
  if (lane == leader) base = atomicAdd(count + b, __popc(ballot));
  base = __shfl_sync(0xffffffffu, base, leader);
  if (on) rows[(long long)b * vr.n_video + base + __popc(ballot & ((1u << lane) - 1u))] = tok;
}

// Row r < count[b] of the compact buffer <- token rows[b][r] of the strided
// tensor (gather), or the reverse (scatter); one warp per row, 16-byte
// accesses.  Strides are in 16-byte units.
template <bool GATHER>
__global__ void __launch_bounds__(256) move_rows_kernel(const uint4* __restrict__ src,
                                                        uint4* __restrict__ dst, long long st,
                                                        long long sb, int row_u4, int n_video,
                                                        const int* __restrict__ count,
                                                        const int* __restrict__ rows) {
  const int b = blockIdx.y;
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (r >= count[b]) return;  // the same for every lane of the warp
  const int lane = threadIdx.x & 31;
  const long long tok = rows[(long long)b * n_video + r];
  const long long strided = b * sb + tok * st;
  const long long compact = ((long long)b * n_video + r) * row_u4;
  const uint4* s = src + (GATHER ? strided : compact);
  uint4* d = dst + (GATHER ? compact : strided);
  for (int c = lane; c < row_u4; c += 32) d[c] = s[c];
}

struct MaskedPlan {
  VideoRows vr;
  size_t count_off, rows_off, qc_off, oc_off, bytes;
};

int plan_masked(const mmdit_tensor_desc& d, const mmdit_layout* L, MaskedPlan& p) {
  int rc = check_layout(L, d.n_tokens);
  if (rc) return rc;
  VideoRows& vr = p.vr;
  vr = VideoRows{};
  int tok = 0, ord = 0, frames = 0, H = -1, W = -1;
  for (int i = 0; i < L->n_seg; ++i) {
    const mmdit_segment& s = L->seg[i];
    if (s.kind == MMDIT_SEG_VIDEO) {
      if (s.order != MMDIT_ORDER_RASTER)
        return fail(MMDIT_EUNSUPPORTED, "masked_joint: video segments must be in raster order");
      if (H >= 0 && (s.H != H || s.W != W))
        return fail(MMDIT_EINVAL, "masked_joint: video segments disagree on H, W");
      H = s.H;
      W = s.W;
      vr.ord0[vr.n_seg] = ord;
      vr.tok0[vr.n_seg] = tok;
      vr.frame0[vr.n_seg] = frames;
      ++vr.n_seg;
      ord += s.n_tokens;
      frames += s.T;
    }
    tok += s.n_tokens;
  }
  vr.hw = H > 0 ? H * W : 1;
  vr.n_video = ord;
  vr.frames = frames;
  const size_t B = (size_t)d.batch, Nv = (size_t)ord, row = (size_t)d.heads * 128 * 2;
  p.count_off = 0;
  p.rows_off = align256(B * sizeof(int));
  p.qc_off = p.rows_off + align256(B * Nv * sizeof(int));
  p.oc_off = p.qc_off + align256(B * Nv * row);
  p.bytes = p.oc_off + align256(B * Nv * row);
  return MMDIT_OK;
}

}  // namespace

}  // namespace mmdit

using namespace mmdit;

extern "C" {

size_t mmdit_masked_joint_attn_workspace_size(const mmdit_tensor_desc* desc,
                                              const mmdit_layout* layout) {
  if (desc == nullptr || check_desc(desc, "masked_joint")) return 0;
  MaskedPlan p;
  if (plan_masked(*desc, layout, p)) return 0;
  return p.bytes;
}

int mmdit_masked_joint_attn(const void* q, const void* k, const void* v, void* o,
                            const mmdit_tensor_desc* desc, const mmdit_layout* layout,
                            float scale, const uint8_t* mask, int64_t mask_elems,
                            void* workspace, size_t ws_bytes, mmdit_stream_t stream) {
  MMDIT_NVTX("mmdit_masked_joint_attn");
  int rc = check_desc(desc, "masked_joint");
  if (rc) return rc;
  if (desc->dtype != MMDIT_BF16) return fail(MMDIT_EUNSUPPORTED, "masked_joint: bf16 only");
  if (!q || !k || !v || !o) return fail(MMDIT_EINVAL, "masked_joint: q, k, v, o must be non-NULL");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return fail(MMDIT_EINVAL, "masked_joint: tensors must be 16-byte aligned");
  if (o == q || o == k || o == v) return fail(MMDIT_EINVAL, "masked_joint: o aliases an input");
  if (!(scale > 0.f) || !isfinite(scale)) return fail(MMDIT_EINVAL, "masked_joint: scale must be > 0");
  if (desc->batch > 65535)  // batch items are grid rows of the row kernels
    return fail(MMDIT_EINVAL, "masked_joint: batch %d > 65535", desc->batch);
  MaskedPlan p;
  if ((rc = plan_masked(*desc, layout, p))) return rc;
  const long long expect = (long long)desc->batch * p.vr.frames * p.vr.hw;
  if (mask_elems != (p.vr.n_video > 0 ? expect : 0))
    return fail(MMDIT_EINVAL, "masked_joint: mask has %lld elements, expected B*F*H*W = %lld",
                (long long)mask_elems, p.vr.n_video > 0 ? expect : 0LL);
  if (p.vr.n_video == 0 || desc->n_tokens == 0) return MMDIT_OK;  // no video row to refine
  if (mask == nullptr) return fail(MMDIT_EINVAL, "masked_joint: mask is NULL");
  if (workspace == nullptr || ws_bytes < p.bytes)
    return fail(MMDIT_EWORKSPACE, "masked_joint: workspace needs %zu bytes", p.bytes);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(MMDIT_EINVAL, "masked_joint: workspace must be 256-byte aligned");
  if ((rc = check_sm100())) return rc;
  int* err = device_error_flag();
  if (err == nullptr) return fail(MMDIT_ECUDA, "device error flag unavailable");

  char* ws = static_cast<char*>(workspace);
  int* count = reinterpret_cast<int*>(ws + p.count_off);
  int* rows = reinterpret_cast<int*>(ws + p.rows_off);
  void* qc = ws + p.qc_off;
  void* oc = ws + p.oc_off;
  const int B = desc->batch, Nv = p.vr.n_video;
  // the compact rows as a [B, Nv, H, 128] tensor
  mmdit_tensor_desc cd = *desc;
  cd.n_tokens = Nv;
  cd.stride_tok = (long long)desc->heads * 128;
  cd.stride_batch = cd.stride_tok * Nv;

  AttnParams ap{};
  AttnProblem& pr = ap.prob;
  if ((rc = make_map(&pr.tmQ, qc, cd, Nv, "masked q")) ||
      (rc = make_map(&pr.tmK, k, *desc, desc->n_tokens, "k")) ||
      (rc = make_map(&pr.tmV, v, *desc, desc->n_tokens, "v")) ||
      (rc = make_store_map(&pr.tmO, oc, cd, Nv, attn_store_cols(2), "masked o")))
    return rc;
  pr.o = (__nv_bfloat16*)oc;
  pr.o_st = cd.stride_tok;
  pr.o_sb = cd.stride_batch;
  pr.Nq = Nv;
  pr.Nkv = desc->n_tokens;
  pr.H = desc->heads;
  pr.B = B;
  pr.n_qtiles = (Nv + 255) / 256;
  pr.n_splits = 1;
  pr.kv_per_split = ((desc->n_tokens + 127) / 128) * 128;
  pr.ctas = pr.n_qtiles * pr.H * pr.B;
  pr.q_count = count;
  ap.q_tiles = 2;
  ap.persistent = 0;
  ap.scale_log2 = scale * 1.4426950408889634f;
  ap.err = err;

  cudaStream_t s = (cudaStream_t)stream;
  const int row_u4 = desc->heads * 16;  // 128 bf16 per head = 16 x 16 bytes
  cudaError_t e = cudaMemsetAsync(count, 0, sizeof(int) * B, s);
  if (e == cudaSuccess) {
    mask_rows_kernel<<<dim3((Nv + 255) / 256, B), 256, 0, s>>>(mask, p.vr, count, rows);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) {
    move_rows_kernel<true><<<dim3((Nv + 7) / 8, B), 256, 0, s>>>(
        static_cast<const uint4*>(q), static_cast<uint4*>(qc), desc->stride_tok / 8,
        desc->stride_batch / 8, row_u4, Nv, count, rows);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) e = launch_attn_tc(ap, s);
  if (e == cudaSuccess) {
    move_rows_kernel<false><<<dim3((Nv + 7) / 8, B), 256, 0, s>>>(
        static_cast<const uint4*>(oc), static_cast<uint4*>(o), desc->stride_tok / 8,
        desc->stride_batch / 8, row_u4, Nv, count, rows);
    e = cudaGetLastError();
  }
  return e == cudaSuccess ? MMDIT_OK : cuda_fail(e, "masked_joint launch");
}

}  // extern "C"
