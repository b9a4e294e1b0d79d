// C-ABI front end of the library (declared in include/mmdit.h): argument
// validation, TMA tensor-map encoding and kernel launches.  Every argument is
// checked before anything is launched; no call allocates device memory.
#include <cudaTypedefs.h>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>

#include <mutex>
#include <string>

#include "internal.h"

namespace mmdit {

__device__ int g_device_error_word = 0;

namespace {
thread_local std::string t_last_error;
}  // namespace

// Helpers below are shared with the other entry-point file (noalloc.cu)
// through internal.h.

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(MMDIT_ECUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_desc(const mmdit_tensor_desc* d, const char* name) {
  if (d == nullptr) return fail(MMDIT_EINVAL, "%s: descriptor is NULL", name);
  if (d->batch < 1 || d->n_tokens < 0 || d->heads < 1)
    return fail(MMDIT_EINVAL, "%s: batch=%d n_tokens=%d heads=%d out of range", name, d->batch,
                d->n_tokens, d->heads);
  if (d->dtype != MMDIT_BF16 && d->dtype != MMDIT_F32)
    return fail(MMDIT_EUNSUPPORTED, "%s: dtype %d not supported", name, d->dtype);
  if (d->dtype == MMDIT_BF16 && d->head_dim != 128)
    return fail(MMDIT_EUNSUPPORTED, "%s: bf16 needs head_dim 128 (got %d)", name, d->head_dim);
  if (d->dtype == MMDIT_F32 && d->head_dim != 64 && d->head_dim != 128)
    return fail(MMDIT_EUNSUPPORTED, "%s: f32 needs head_dim 64 or 128 (got %d)", name,
                d->head_dim);
  const long long row = (long long)d->heads * d->head_dim;
  if (d->stride_tok < row)
    return fail(MMDIT_EINVAL, "%s: stride_tok %lld < heads*head_dim %lld", name, d->stride_tok, row);
  if (d->batch > 1 && d->stride_batch < d->stride_tok * (long long)d->n_tokens)
    return fail(MMDIT_EINVAL, "%s: stride_batch %lld overlaps batch items", name, d->stride_batch);
  const int es = d->dtype == MMDIT_BF16 ? 2 : 4;
  if ((d->stride_tok * es) % 16 != 0 || (d->stride_batch * es) % 16 != 0)
    return fail(MMDIT_EINVAL, "%s: strides must be multiples of 16 bytes", name);
  return MMDIT_OK;
}

int check_layout(const mmdit_layout* L, int n_tokens) {
  if (L == nullptr) return fail(MMDIT_EINVAL, "layout is NULL");
  if (L->n_seg < 1 || L->n_seg > MMDIT_MAX_SEGMENTS)
    return fail(MMDIT_EINVAL, "layout: n_seg %d outside [1, %d]", L->n_seg, MMDIT_MAX_SEGMENTS);
  long long total = 0;
  for (int i = 0; i < L->n_seg; ++i) {
    const mmdit_segment& s = L->seg[i];
    if (s.n_tokens < 0) return fail(MMDIT_EINVAL, "layout: segment %d has n_tokens < 0", i);
    if (s.kind == MMDIT_SEG_VIDEO) {
      if (s.T < 1 || s.H < 1 || s.W < 1 || (long long)s.T * s.H * s.W != s.n_tokens)
        return fail(MMDIT_EINVAL, "layout: video segment %d: T*H*W != n_tokens", i);
      if (s.order != MMDIT_ORDER_RASTER && s.order != MMDIT_ORDER_BLOCK444)
        return fail(MMDIT_EINVAL, "layout: segment %d: bad order %d", i, s.order);
    } else if (s.kind == MMDIT_SEG_AUDIO) {
      if (s.t_den < 1 || s.t_num < 0 || (long long)s.n_tokens * s.t_num > 0x7fffffffLL)
        return fail(MMDIT_EINVAL, "layout: audio segment %d: bad t_num/t_den", i);
    } else if (s.kind != MMDIT_SEG_TEXT) {
      return fail(MMDIT_EINVAL, "layout: segment %d: bad kind %d", i, s.kind);
    }
    total += s.n_tokens;
  }
  if (total != n_tokens)
    return fail(MMDIT_EINVAL, "layout: segments hold %lld tokens, tensor has %d", total, n_tokens);
  return MMDIT_OK;
}

DevLayout to_dev(const mmdit_layout* L) {
  DevLayout d{};
  d.n_seg = L->n_seg;
  int start = 0;
  for (int i = 0; i < L->n_seg; ++i) {
    const mmdit_segment& s = L->seg[i];
    d.seg[i] = DevSeg{s.kind, start, s.n_tokens, s.T, s.H, s.W, s.t0, s.t_num, s.t_den, s.order};
    start += s.n_tokens;
  }
  return d;
}

int make_rope_tab(const mmdit_rope_params* r, int head_dim, RopeTab& tab) {
  if (r == nullptr) return fail(MMDIT_EINVAL, "rope parameters are NULL");
  if (!(r->theta > 0.f) || r->dim_t < 0 || r->dim_h < 0 || r->dim_w < 0 || (r->dim_t & 1) ||
      (r->dim_h & 1) || (r->dim_w & 1) || r->dim_t + r->dim_h + r->dim_w != head_dim)
    return fail(MMDIT_EINVAL, "rope: need theta > 0 and even dims summing to head_dim %d",
                head_dim);
  tab = RopeTab{};
  tab.pt = r->dim_t / 2;
  tab.ph = (r->dim_t + r->dim_h) / 2;
  tab.npairs = head_dim / 2;
  const int dims[3] = {r->dim_t, r->dim_h, r->dim_w};
  int m = 0;
  for (int a = 0; a < 3; ++a)
    for (int i = 0; i < dims[a] / 2; ++i, ++m)
      tab.omega[m] = (float)pow((double)r->theta, -2.0 * i / (double)dims[a]);
  return MMDIT_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 4D map {channel, head, token, batch} over a bf16 [B, N, heads, 128] tensor,
// box {64, 1, 64, 1}, 128-byte swizzle, zero fill out of bounds.
int make_map(CUtensorMap* m, const void* base, const mmdit_tensor_desc& d, int n_tokens,
             const char* name) {
  auto fn = encode_fn();
  if (fn == nullptr) return fail(MMDIT_ECUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[4] = {128, (cuuint64_t)d.heads, (cuuint64_t)n_tokens, (cuuint64_t)d.batch};
  cuuint64_t strides[3] = {128 * 2, (cuuint64_t)d.stride_tok * 2,
                           (cuuint64_t)(d.batch > 1 ? d.stride_batch : d.stride_tok * n_tokens) * 2};
  cuuint32_t box[4] = {64, 1, 64, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MMDIT_ECUDA, "%s: tensor map encoding failed (%d)", name, (int)r);
  return MMDIT_OK;
}

int make_store_map(CUtensorMap* m, void* base, const mmdit_tensor_desc& d, int n_tokens,
                   int cols, const char* name) {
  if (cols != 32 && cols != 64) return fail(MMDIT_EINVAL, "%s: store box of %d channels", name, cols);
  auto fn = encode_fn();
  if (fn == nullptr) return fail(MMDIT_ECUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[4] = {128, (cuuint64_t)d.heads, (cuuint64_t)n_tokens, (cuuint64_t)d.batch};
  cuuint64_t strides[3] = {128 * 2, (cuuint64_t)d.stride_tok * 2,
                           (cuuint64_t)(d.batch > 1 ? d.stride_batch : d.stride_tok * n_tokens) * 2};
  cuuint32_t box[4] = {(cuuint32_t)cols, 1, 32, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, base, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE,
                  cols == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                  CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MMDIT_ECUDA, "%s: tensor map encoding failed (%d)", name, (int)r);
  return MMDIT_OK;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

int check_sm100() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0)
    return fail(MMDIT_EUNSUPPORTED, "device %d is sm_%d%d; this library targets sm_100a", dev,
                major, minor);
  return MMDIT_OK;
}

// Split of the video keys for the audio-query direction: enough splits that
// the (few) audio query tiles x heads x batch fill one wave of the B200's 148
// SMs, each split a whole number of 128-key tiles.  One wave of long items
// measured faster than two waves of half-length items (less pipeline fill and
// drain per key, half the partials to merge).
constexpr int kCrossTargetCtas = 148;

// Q tiles per CTA of video queries over a short key sequence (audio, text):
// one tile, two CTAs per SM (measured faster than two tiles with resident K/V).
constexpr int kShortKvQTiles = 1;

// Q tiles per CTA of the dense joint attention: two, one CTA per SM.
constexpr int kJointQTiles = 2;

CrossPlan plan_cross(const mmdit_tensor_desc* v, const mmdit_tensor_desc* a) {
  CrossPlan p{};
  p.n_qtiles_a = (a->n_tokens + 255) / 256;
  const int tiles = (v->n_tokens + 127) / 128;
  const int base = p.n_qtiles_a * a->heads * a->batch;
  p.splits = std::max(1, std::min(tiles, (kCrossTargetCtas + base / 2) / base));
  p.kv_per_split = ((tiles + p.splits - 1) / p.splits) * 128;
  p.splits = std::max(1, (v->n_tokens + p.kv_per_split - 1) / p.kv_per_split);
  p.nq_pad = p.n_qtiles_a * 256;
  const size_t rows = (size_t)p.splits * a->batch * a->heads * p.nq_pad;
  p.part_o_bytes = align256(rows * 128 * sizeof(float));
  p.part_ml_bytes = align256(rows * 2 * sizeof(float));
  return p;
}

// Video queries over a short key sequence (the audio or the text tokens):
// persistent CTAs of kShortKvQTiles Q tiles (two CTAs per SM for one tile, so
// that each hides the other's load and epilogue latency), all key tiles in one
// work item, bf16 O written through the output tensor map.
int short_kv_params(AttnParams& p, const void* q, const void* k, const void* v, void* o,
                    const mmdit_tensor_desc& qd, const mmdit_tensor_desc& kd, float scale,
                    int* err, const char* qname, const char* kname) {
  int rc;
  AttnProblem& pr = p.prob;
  if ((rc = make_map(&pr.tmQ, q, qd, qd.n_tokens, qname)) ||
      (rc = make_map(&pr.tmK, k, kd, kd.n_tokens, kname)) ||
      (rc = make_map(&pr.tmV, v, kd, kd.n_tokens, kname)) ||
      (rc = make_store_map(&pr.tmO, o, qd, qd.n_tokens, attn_store_cols(kShortKvQTiles), qname)))
    return rc;
  pr.o = (__nv_bfloat16*)o;
  pr.o_st = qd.stride_tok;
  pr.o_sb = qd.stride_batch;
  pr.Nq = qd.n_tokens;
  pr.Nkv = kd.n_tokens;
  pr.H = qd.heads;
  pr.B = qd.batch;
  pr.n_qtiles = (qd.n_tokens + 128 * kShortKvQTiles - 1) / (128 * kShortKvQTiles);
  pr.n_splits = 1;
  pr.kv_per_split = ((kd.n_tokens + 127) / 128) * 128;
  pr.ctas = pr.n_qtiles * pr.H * pr.B;
  p.q_tiles = kShortKvQTiles;
  p.persistent = 1;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.err = err;
  return MMDIT_OK;
}

int launch_cross(const void* qv, const void* kv, const void* vv, const void* qa, const void* ka,
                 const void* va, void* o_video, void* o_audio, const mmdit_tensor_desc& video,
                 const mmdit_tensor_desc& audio, float scale, int splits, int kv_per_split,
                 float* part_o, float* part_ml, cudaStream_t s, float* row_sq,
                 float* video_norm) {
  int rc;
  int* err = device_error_flag();
  if (err == nullptr) return fail(MMDIT_ECUDA, "device error flag unavailable");
  // audio queries over the video keys: 2 Q tiles per CTA, keys split across
  // CTAs, unnormalised partials merged by the combine kernel
  AttnParams pa{};
  AttnProblem& a2v = pa.prob;
  if ((rc = make_map(&a2v.tmQ, qa, audio, audio.n_tokens, "qa")) ||
      (rc = make_map(&a2v.tmK, kv, video, video.n_tokens, "kv")) ||
      (rc = make_map(&a2v.tmV, vv, video, video.n_tokens, "vv")))
    return rc;
  a2v.o = nullptr;
  a2v.part_o = part_o;
  a2v.part_ml = part_ml;
  a2v.Nq = audio.n_tokens;
  a2v.Nkv = video.n_tokens;
  a2v.H = audio.heads;
  a2v.B = audio.batch;
  a2v.n_qtiles = (audio.n_tokens + 255) / 256;
  a2v.n_splits = splits;
  a2v.kv_per_split = kv_per_split;
  a2v.ctas = a2v.n_qtiles * a2v.n_splits * a2v.H * a2v.B;
  pa.q_tiles = 2;
  pa.persistent = 1;
  pa.scale_log2 = scale * 1.4426950408889634f;
  pa.err = err;
  // video queries over the (short) audio keys
  AttnParams pv{};
  if ((rc = short_kv_params(pv, qv, ka, va, o_video, video, audio, scale, err, "video", "audio")))
    return rc;
  pv.prob.row_sq = video_norm != nullptr ? row_sq : nullptr;
  cudaError_t e = launch_attn_tc(pa, s);
  // video queries: every audio key in one tile when there are at most 256
  if (e == cudaSuccess)
    e = audio.n_tokens <= kShortKeys ? launch_attn_short(pv, s) : launch_attn_tc(pv, s);
  if (e == cudaSuccess)
    e = launch_split_combine(part_o, part_ml, (__nv_bfloat16*)o_audio, audio.stride_tok,
                             audio.stride_batch, splits, audio.batch, audio.heads, audio.n_tokens,
                             a2v.n_qtiles * 256, s);
  if (e == cudaSuccess && video_norm != nullptr)
    e = launch_cross_norms(row_sq, video.heads, (long long)video.batch * video.n_tokens,
                           video_norm, s);
  return e == cudaSuccess ? MMDIT_OK : cuda_fail(e, "av_cross launch");
}

int* device_error_flag() {
  static std::atomic<int*> cache[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  int* p = cache[dev].load(std::memory_order_acquire);
  if (p != nullptr) return p;
  std::lock_guard<std::mutex> lock(mu);
  p = cache[dev].load(std::memory_order_relaxed);
  if (p == nullptr) {
    void* a = nullptr;
    if (cudaGetSymbolAddress(&a, g_device_error_word) != cudaSuccess) return nullptr;
    p = static_cast<int*>(a);
    cache[dev].store(p, std::memory_order_release);
  }
  return p;
}

}  // namespace mmdit

using namespace mmdit;

extern "C" {

const char* mmdit_last_error(void) { return t_last_error.c_str(); }

const char* mmdit_version(void) { return "mmdit-av-attn 0.1.0 (sm_100a)"; }

int mmdit_device_status(mmdit_stream_t stream) {
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_device_error_word, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "reading the device error flag");
  if (v != 0) {
    const int zero = 0;
    cudaMemcpyToSymbol(g_device_error_word, &zero, sizeof(int));
    return fail(v, v == MMDIT_EDEVCHECK ? "a device-side index check failed (status %d)"
                                        : "a bounded device wait ran out (status %d)",
                v);
  }
  return MMDIT_OK;
}

int mmdit_rope_apply(void* q, void* k, const mmdit_tensor_desc* desc, const mmdit_layout* layout,
                     const mmdit_rope_params* rope, mmdit_stream_t stream) {
  MMDIT_NVTX("mmdit_rope_apply");
  int rc = check_desc(desc, "rope");
  if (rc) return rc;
  if (q == nullptr && k == nullptr) return fail(MMDIT_EINVAL, "rope: q and k are both NULL");
  if ((q && !aligned16(q)) || (k && !aligned16(k)))
    return fail(MMDIT_EINVAL, "rope: tensors must be 16-byte aligned");
  if ((rc = check_layout(layout, desc->n_tokens))) return rc;
  RopeTab tab;
  if ((rc = make_rope_tab(rope, desc->head_dim, tab))) return rc;
  if (desc->n_tokens == 0) return MMDIT_OK;
  cudaError_t e = launch_rope(q, k, *desc, to_dev(layout), tab, (cudaStream_t)stream);
  return e == cudaSuccess ? MMDIT_OK : cuda_fail(e, "rope launch");
}

size_t mmdit_joint_attn_workspace_size(const mmdit_tensor_desc*) { return 0; }

int mmdit_joint_attn(const void* q, const void* k, const void* v, void* o, float* lse,
                     const mmdit_tensor_desc* desc, const mmdit_layout* layout, float scale,
                     const mmdit_rope_params* rope_q, const uint8_t* cond_mask, int64_t mask_elems,
                     void*, size_t, mmdit_stream_t stream) {
  MMDIT_NVTX("mmdit_joint_attn");
  int rc = check_desc(desc, "joint_attn");
  if (rc) return rc;
  if (!q || !k || !v || !o) return fail(MMDIT_EINVAL, "joint_attn: q, k, v, o must be non-NULL");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return fail(MMDIT_EINVAL, "joint_attn: tensors must be 16-byte aligned");
  if (o == q || o == k || o == v) return fail(MMDIT_EINVAL, "joint_attn: o aliases an input");
  if (!(scale > 0.f) || !isfinite(scale)) return fail(MMDIT_EINVAL, "joint_attn: scale must be > 0");
  if ((rc = check_layout(layout, desc->n_tokens))) return rc;
  if (cond_mask != nullptr) {
    // the channel-concat mask M: carried with the inputs, never applied
    long long frames = 0;
    int mh = -1, mw = -1;
    for (int i = 0; i < layout->n_seg; ++i) {
      const mmdit_segment& s = layout->seg[i];
      if (s.kind != MMDIT_SEG_VIDEO) continue;
      if (mh >= 0 && (s.H != mh || s.W != mw))
        return fail(MMDIT_EINVAL, "joint_attn: video segments disagree on H, W for the mask");
      mh = s.H;
      mw = s.W;
      frames += s.T;
    }
    const long long expect = mh < 0 ? 0 : (long long)desc->batch * frames * mh * mw;
    if (mask_elems != expect)
      return fail(MMDIT_EINVAL, "joint_attn: mask has %lld elements, expected B*F*H*W = %lld",
                  (long long)mask_elems, expect);
  }
  RopeTab tab{};
  if (rope_q != nullptr) {
    if (desc->dtype != MMDIT_BF16)
      return fail(MMDIT_EUNSUPPORTED, "joint_attn: fused Q RoPE needs bf16");
    if ((rc = make_rope_tab(rope_q, desc->head_dim, tab))) return rc;
  }
  if (desc->n_tokens == 0) return MMDIT_OK;
  if (desc->dtype == MMDIT_F32) {
    F32AttnArgs a{(const float*)q, (const float*)k, (const float*)v, (float*)o, lse,
                  desc->batch, desc->heads, desc->head_dim, desc->n_tokens, desc->n_tokens,
                  desc->stride_tok, desc->stride_batch, desc->stride_tok, desc->stride_batch,
                  desc->stride_tok, desc->stride_batch, desc->stride_tok, desc->stride_batch, scale};
    cudaError_t e = launch_attn_f32(a, (cudaStream_t)stream);
    return e == cudaSuccess ? MMDIT_OK : cuda_fail(e, "attn_f32 launch");
  }
  if ((rc = check_sm100())) return rc;
  AttnParams p{};
  AttnProblem& pr = p.prob;
  if ((rc = make_map(&pr.tmQ, q, *desc, desc->n_tokens, "q")) ||
      (rc = make_map(&pr.tmK, k, *desc, desc->n_tokens, "k")) ||
      (rc = make_map(&pr.tmV, v, *desc, desc->n_tokens, "v")))
    return rc;
  if ((rc = make_store_map(&pr.tmO, o, *desc, desc->n_tokens, attn_store_cols(kJointQTiles), "o"))) return rc;
  pr.o = (__nv_bfloat16*)o;
  pr.o_st = desc->stride_tok;
  pr.o_sb = desc->stride_batch;
  pr.lse = lse;
  pr.Nq = pr.Nkv = desc->n_tokens;
  pr.H = desc->heads;
  pr.B = desc->batch;
  pr.n_qtiles = (desc->n_tokens + 255) / 256;
  pr.n_splits = 1;
  pr.kv_per_split = ((desc->n_tokens + 127) / 128) * 128;
  pr.ctas = pr.n_qtiles * pr.H * pr.B;
  pr.rope_q = rope_q != nullptr;
  p.q_tiles = kJointQTiles;
  p.persistent = 0;  // measured: one item per CTA is ~1% faster for long keys
  p.scale_log2 = scale * 1.4426950408889634f;
  p.layout = to_dev(layout);
  p.rope = tab;
  p.err = device_error_flag();
  if (p.err == nullptr) return fail(MMDIT_ECUDA, "device error flag unavailable");
  cudaError_t e = launch_attn_tc(p, (cudaStream_t)stream);
  return e == cudaSuccess ? MMDIT_OK : cuda_fail(e, "attn_tc launch");
}

size_t mmdit_av_cross_attn_workspace_size(const mmdit_tensor_desc* video,
                                          const mmdit_tensor_desc* audio) {
  if (video == nullptr || audio == nullptr || video->dtype != MMDIT_BF16) return 0;
  if (check_desc(video, "video") || check_desc(audio, "audio")) return 0;
  const CrossPlan c = plan_cross(video, audio);
  return c.part_o_bytes + c.part_ml_bytes;
}

int mmdit_av_cross_attn(const void* qv, const void* kv, const void* vv, const void* qa,
                        const void* ka, const void* va, void* o_video, void* o_audio,
                        const mmdit_tensor_desc* video, const mmdit_tensor_desc* audio,
                        float scale, void* workspace, size_t ws_bytes, mmdit_stream_t stream) {
  MMDIT_NVTX("mmdit_av_cross_attn");
  int rc;
  if ((rc = check_desc(video, "video")) || (rc = check_desc(audio, "audio"))) return rc;
  if (video->batch != audio->batch || video->heads != audio->heads ||
      video->head_dim != audio->head_dim || video->dtype != audio->dtype)
    return fail(MMDIT_EINVAL, "av_cross: video and audio descriptors disagree");
  const void* ptrs[8] = {qv, kv, vv, qa, ka, va, o_video, o_audio};
  for (const void* p : ptrs) {
    if (p == nullptr) return fail(MMDIT_EINVAL, "av_cross: every tensor must be non-NULL");
    if (!aligned16(p)) return fail(MMDIT_EINVAL, "av_cross: tensors must be 16-byte aligned");
  }
  if (video->n_tokens < 1 || audio->n_tokens < 1)
    return fail(MMDIT_EINVAL, "av_cross: both streams need at least one token");
  if (!(scale > 0.f) || !isfinite(scale)) return fail(MMDIT_EINVAL, "av_cross: scale must be > 0");
  cudaStream_t s = (cudaStream_t)stream;
  if (video->dtype == MMDIT_F32) {
    F32AttnArgs a1{(const float*)qv, (const float*)ka, (const float*)va, (float*)o_video, nullptr,
                   video->batch, video->heads, video->head_dim, video->n_tokens, audio->n_tokens,
                   video->stride_tok, video->stride_batch, audio->stride_tok, audio->stride_batch,
                   audio->stride_tok, audio->stride_batch, video->stride_tok, video->stride_batch,
                   scale};
    F32AttnArgs a2{(const float*)qa, (const float*)kv, (const float*)vv, (float*)o_audio, nullptr,
                   audio->batch, audio->heads, audio->head_dim, audio->n_tokens, video->n_tokens,
                   audio->stride_tok, audio->stride_batch, video->stride_tok, video->stride_batch,
                   video->stride_tok, video->stride_batch, audio->stride_tok, audio->stride_batch,
                   scale};
    cudaError_t e = launch_attn_f32(a1, s);
    if (e == cudaSuccess) e = launch_attn_f32(a2, s);
    return e == cudaSuccess ? MMDIT_OK : cuda_fail(e, "attn_f32 launch");
  }
  const CrossPlan c = plan_cross(video, audio);
  if (workspace == nullptr || ws_bytes < c.part_o_bytes + c.part_ml_bytes)
    return fail(MMDIT_EWORKSPACE, "av_cross: workspace needs %zu bytes", c.part_o_bytes + c.part_ml_bytes);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(MMDIT_EINVAL, "av_cross: workspace must be 256-byte aligned");
  if ((rc = check_sm100())) return rc;
  return launch_cross(qv, kv, vv, qa, ka, va, o_video, o_audio, *video, *audio, scale, c.splits,
                      c.kv_per_split, reinterpret_cast<float*>(workspace),
                      reinterpret_cast<float*>(static_cast<char*>(workspace) + c.part_o_bytes), s);
}

size_t mmdit_av_cross_attn_norms_workspace_size(const mmdit_tensor_desc* video,
                                                const mmdit_tensor_desc* audio) {
  const size_t base = mmdit_av_cross_attn_workspace_size(video, audio);
  if (base == 0) return 0;
  return base + align256(sizeof(float) * (size_t)video->batch * video->n_tokens * video->heads);
}

int mmdit_av_cross_attn_norms(const void* qv, const void* kv, const void* vv, const void* qa,
                              const void* ka, const void* va, void* o_video, void* o_audio,
                              const mmdit_tensor_desc* video, const mmdit_tensor_desc* audio,
                              float scale, float* video_norm, void* workspace, size_t ws_bytes,
                              mmdit_stream_t stream) {
  MMDIT_NVTX("mmdit_av_cross_attn_norms");
  int rc;
  if ((rc = check_desc(video, "video")) || (rc = check_desc(audio, "audio"))) return rc;
  if (video->batch != audio->batch || video->heads != audio->heads ||
      video->head_dim != audio->head_dim || video->dtype != audio->dtype)
    return fail(MMDIT_EINVAL, "av_cross_norms: video and audio descriptors disagree");
  if (video->dtype != MMDIT_BF16) return fail(MMDIT_EUNSUPPORTED, "av_cross_norms: bf16 only");
  const void* ptrs[8] = {qv, kv, vv, qa, ka, va, o_video, o_audio};
  for (const void* p : ptrs) {
    if (p == nullptr) return fail(MMDIT_EINVAL, "av_cross_norms: every tensor must be non-NULL");
    if (!aligned16(p)) return fail(MMDIT_EINVAL, "av_cross_norms: tensors must be 16-byte aligned");
  }
  if (video_norm == nullptr || (reinterpret_cast<uintptr_t>(video_norm) & 3u))
    return fail(MMDIT_EINVAL, "av_cross_norms: video_norm must be an aligned device float array");
  if (video->n_tokens < 1 || audio->n_tokens < 1)
    return fail(MMDIT_EINVAL, "av_cross_norms: both streams need at least one token");
  if (!(scale > 0.f) || !isfinite(scale)) return fail(MMDIT_EINVAL, "av_cross_norms: scale must be > 0");
  const CrossPlan c = plan_cross(video, audio);
  const size_t need = mmdit_av_cross_attn_norms_workspace_size(video, audio);
  if (workspace == nullptr || ws_bytes < need)
    return fail(MMDIT_EWORKSPACE, "av_cross_norms: workspace needs %zu bytes", need);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(MMDIT_EINVAL, "av_cross_norms: workspace must be 256-byte aligned");
  if ((rc = check_sm100())) return rc;
  char* ws = static_cast<char*>(workspace);
  return launch_cross(qv, kv, vv, qa, ka, va, o_video, o_audio, *video, *audio, scale, c.splits,
                      c.kv_per_split, reinterpret_cast<float*>(ws),
                      reinterpret_cast<float*>(ws + c.part_o_bytes), (cudaStream_t)stream,
                      reinterpret_cast<float*>(ws + c.part_o_bytes + c.part_ml_bytes), video_norm);
}

int mmdit_text_cross_attn(const void* qv, const void* kt, const void* vt, void* o_video,
                          const mmdit_tensor_desc* video, const mmdit_tensor_desc* text,
                          float scale, mmdit_stream_t stream) {
  MMDIT_NVTX("mmdit_text_cross_attn");
  int rc;
  if ((rc = check_desc(video, "video")) || (rc = check_desc(text, "text"))) return rc;
  if (video->batch != text->batch || video->heads != text->heads ||
      video->head_dim != text->head_dim || video->dtype != text->dtype)
    return fail(MMDIT_EINVAL, "text_cross: video and text descriptors disagree");
  const void* ptrs[4] = {qv, kt, vt, o_video};
  for (const void* p : ptrs) {
    if (p == nullptr) return fail(MMDIT_EINVAL, "text_cross: every tensor must be non-NULL");
    if (!aligned16(p)) return fail(MMDIT_EINVAL, "text_cross: tensors must be 16-byte aligned");
  }
  if (o_video == qv) return fail(MMDIT_EINVAL, "text_cross: o_video aliases qv");
  if (text->n_tokens < 1) return fail(MMDIT_EINVAL, "text_cross: at least one text token");
  if (!(scale > 0.f) || !isfinite(scale)) return fail(MMDIT_EINVAL, "text_cross: scale must be > 0");
  if (video->n_tokens == 0) return MMDIT_OK;
  cudaStream_t s = (cudaStream_t)stream;
  if (video->dtype == MMDIT_F32) {
    F32AttnArgs a{(const float*)qv, (const float*)kt, (const float*)vt, (float*)o_video, nullptr,
                  video->batch, video->heads, video->head_dim, video->n_tokens, text->n_tokens,
                  video->stride_tok, video->stride_batch, text->stride_tok, text->stride_batch,
                  text->stride_tok, text->stride_batch, video->stride_tok, video->stride_batch,
                  scale};
    cudaError_t e = launch_attn_f32(a, s);
    return e == cudaSuccess ? MMDIT_OK : cuda_fail(e, "attn_f32 launch");
  }
  if ((rc = check_sm100())) return rc;
  int* err = device_error_flag();
  if (err == nullptr) return fail(MMDIT_ECUDA, "device error flag unavailable");
  AttnParams p{};
  if ((rc = short_kv_params(p, qv, kt, vt, o_video, *video, *text, scale, err, "video", "text")))
    return rc;
  cudaError_t e = launch_attn_tc(p, s);
  return e == cudaSuccess ? MMDIT_OK : cuda_fail(e, "text_cross launch");
}

}  // extern "C"
