// Allocation-free variant of the audio<->video cross-attention.
//
// The regular mmdit_av_cross_attn needs a caller-sized workspace for the
// split-KV partial results of the audio-query direction.  Some callers cannot
// provide one: a plugin hosted by an inference runtime that owns every device
// allocation of the process, or a serving loop that forbids allocation after
// start-up so that its memory footprint stays fixed, has no way to call
// cudaMalloc or to grow a workspace on demand.  mmdit_av_cross_attn_noalloc
// serves them: its scratch is a fixed file-scope device array of
// MMDIT_NOALLOC_SCRATCH_BYTES, so the call allocates nothing.  Every GPU that
// loads this library holds that array until the process exits.
//
// The array is a device symbol.  Host code cannot use its name as an address
// (a kernel handed the host-side stand-in would fault or, where the GPU can
// reach host memory, silently use the wrong memory), so the first call on each
// device, with that device current, looks the address up once with
// cudaGetSymbolAddress and caches it; that first call should therefore come
// before any stream capture.  Every call shares the array and finds the
// previous call's contents in it; nothing here needs it zeroed (every partial
// row is written before it is read).  Calls that overlap on the GPU (two
// streams, or two host threads on one device) race on the array.
#include <mutex>

#include "internal.h"

namespace mmdit {

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[MMDIT_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch on the current device (looked up once
// per device).
int scratch_address(void** out) {
  static void* cache[64] = {};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(MMDIT_EUNSUPPORTED, "device index %d >= 64", dev);
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(noalloc scratch)");
    cache[dev] = p;
  }
  *out = cache[dev];
  return MMDIT_OK;
}

}  // namespace

}  // namespace mmdit

using namespace mmdit;

extern "C" int mmdit_av_cross_attn_noalloc(const void* qv, const void* kv, const void* vv,
                                           const void* qa, const void* ka, const void* va,
                                           void* o_video, void* o_audio,
                                           const mmdit_tensor_desc* video,
                                           const mmdit_tensor_desc* audio, float scale,
                                           mmdit_stream_t stream) {
  MMDIT_NVTX("mmdit_av_cross_attn_noalloc");
  int rc;
  if ((rc = check_desc(video, "video")) || (rc = check_desc(audio, "audio"))) return rc;
  if (video->batch != audio->batch || video->heads != audio->heads ||
      video->head_dim != audio->head_dim || video->dtype != audio->dtype)
    return fail(MMDIT_EINVAL, "av_cross_noalloc: video and audio descriptors disagree");
  if (video->dtype != MMDIT_BF16)
    return fail(MMDIT_EUNSUPPORTED, "av_cross_noalloc: bf16 only");
  const void* ptrs[8] = {qv, kv, vv, qa, ka, va, o_video, o_audio};
  for (const void* p : ptrs) {
    if (p == nullptr) return fail(MMDIT_EINVAL, "av_cross_noalloc: every tensor must be non-NULL");
    if (!aligned16(p)) return fail(MMDIT_EINVAL, "av_cross_noalloc: 16-byte alignment");
  }
  if (video->n_tokens < 1 || audio->n_tokens < 1)
    return fail(MMDIT_EINVAL, "av_cross_noalloc: both streams need at least one token");
  if (!(scale > 0.f) || !isfinite(scale))
    return fail(MMDIT_EINVAL, "av_cross_noalloc: scale must be > 0");

  // Start from the split of the video keys that the regular call uses (one
  // wave of audio-query items over the SMs), then lower the split count until
  // the partial results fit the fixed scratch array.
  const CrossPlan plan = plan_cross(video, audio);
  const int tiles = (video->n_tokens + 127) / 128;
  const size_t rows_per_split = (size_t)audio->batch * audio->heads * plan.nq_pad;
  auto bytes_for = [&](int splits) {
    return align256((size_t)splits * rows_per_split * 128 * sizeof(float)) +
           align256((size_t)splits * rows_per_split * 2 * sizeof(float));
  };
  int splits = plan.splits;
  while (splits > 1 && bytes_for(splits) > (size_t)MMDIT_NOALLOC_SCRATCH_BYTES) --splits;
  if (bytes_for(splits) > (size_t)MMDIT_NOALLOC_SCRATCH_BYTES)
    return fail(MMDIT_EINVAL,
                "av_cross_noalloc: batch*heads*audio rows need %zu bytes of scratch; the "
                "fixed maximum is %d bytes (use mmdit_av_cross_attn with a workspace)",
                bytes_for(1), MMDIT_NOALLOC_SCRATCH_BYTES);
  const int kv_per_split = ((tiles + splits - 1) / splits) * 128;
  splits = (video->n_tokens + kv_per_split - 1) / kv_per_split;
  if ((rc = check_sm100())) return rc;
  void* scratch = nullptr;
  if ((rc = scratch_address(&scratch))) return rc;

  float* part_o = static_cast<float*>(scratch);
  float* part_ml = reinterpret_cast<float*>(
      static_cast<char*>(scratch) + align256((size_t)splits * rows_per_split * 128 * sizeof(float)));
  return launch_cross(qv, kv, vv, qa, ka, va, o_video, o_audio, *video, *audio, scale, splits,
                      kv_per_split, part_o, part_ml, (cudaStream_t)stream);
}
