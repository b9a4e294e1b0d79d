// 3D RoPE over (t, h, w) token positions, applied in place to Q and/or K.
//
// SkyReels-V4 digest (arXiv 2602.21818), novelty 4 (time-offset 3D RoPE:
// conditioning latents carry negative temporal indices) and novelty 5 (audio
// RoPE frequency scaling 21/218); SkyReels-V4 blog (trdm.cn) section 2.2.
// Channels form bands [t | h | w]; the interleaved pair (2i, 2i+1) of band b
// (i counted from the band start) turns by pos_b * theta^(-2i/d_b).
//
// The op is HBM-bound (one read and one write of Q and K).  The rotation angle
// depends on the token and the channel pair only, so each thread owns one
// 16-byte chunk of channels of one token, computes that chunk's sin/cos once,
// and streams the chunk through every head of Q and K.  Loads and stores are
// 16-byte vectors; a warp covers whole 256-byte (bf16, d=128) head rows.
#include "internal.h"

namespace mmdit {

namespace {

template <typename T>
struct Vec;
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int kElems = 8;  // 16 bytes
};
template <>
struct Vec<float> {
  static constexpr int kElems = 4;
};

__device__ __forceinline__ void rot_chunk(uint4& raw, const float* c, const float* s,
                                          __nv_bfloat16*) {
  __nv_bfloat162* p = reinterpret_cast<__nv_bfloat162*>(&raw);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 x = __bfloat1622float2(p[i]);
    float2 y;
    y.x = x.x * c[i] - x.y * s[i];
    y.y = x.x * s[i] + x.y * c[i];
    p[i] = __float22bfloat162_rn(y);
  }
}
__device__ __forceinline__ void rot_chunk(uint4& raw, const float* c, const float* s, float*) {
  float* p = reinterpret_cast<float*>(&raw);
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float x0 = p[2 * i], x1 = p[2 * i + 1];
    p[2 * i] = x0 * c[i] - x1 * s[i];
    p[2 * i + 1] = x0 * s[i] + x1 * c[i];
  }
}

template <typename T>
__global__ void __launch_bounds__(256) rope_kernel(T* __restrict__ q, T* __restrict__ k, int N,
                                                   int H, int D, long long st, long long sb,
                                                   DevLayout L, RopeTab tab) {
  constexpr int E = Vec<T>::kElems;
  constexpr int P = E / 2;  // channel pairs per chunk
  const int cpr = D / E;    // chunks per head row
  const int tpb = blockDim.x / cpr;
  const int tok = blockIdx.x * tpb + threadIdx.x / cpr;
  const int chunk = threadIdx.x % cpr;
  const int b = blockIdx.y;
  if (tok >= N) return;

  float pt, ph, pw;
  token_position(L, tok, pt, ph, pw);
  float cs[P], sn[P];
#pragma unroll
  for (int i = 0; i < P; ++i) {
    const int m = chunk * P + i;
    const float pos = m < tab.pt ? pt : (m < tab.ph ? ph : pw);
    sincosf(pos * tab.omega[m], &sn[i], &cs[i]);
  }
  const long long base = (long long)b * sb + (long long)tok * st + chunk * E;
#pragma unroll 4
  for (int h = 0; h < H; ++h) {
    const long long off = base + (long long)h * D;
    if (q) {
      uint4 v = *reinterpret_cast<const uint4*>(q + off);
      rot_chunk(v, cs, sn, (T*)nullptr);
      *reinterpret_cast<uint4*>(q + off) = v;
    }
    if (k) {
      uint4 v = *reinterpret_cast<const uint4*>(k + off);
      rot_chunk(v, cs, sn, (T*)nullptr);
      *reinterpret_cast<uint4*>(k + off) = v;
    }
  }
}

}  // namespace

cudaError_t launch_rope(void* q, void* k, const mmdit_tensor_desc& d, const DevLayout& L,
                        const RopeTab& tab, cudaStream_t s) {
  if (d.n_tokens == 0) return cudaSuccess;
  const int threads = 256;
  if (d.dtype == MMDIT_BF16) {
    const int cpr = d.head_dim / 8;
    const int tpb = threads / cpr;
    dim3 grid((d.n_tokens + tpb - 1) / tpb, d.batch);
    rope_kernel<__nv_bfloat16><<<grid, threads, 0, s>>>(
        (__nv_bfloat16*)q, (__nv_bfloat16*)k, d.n_tokens, d.heads, d.head_dim, d.stride_tok,
        d.stride_batch, L, tab);
  } else {
    const int cpr = d.head_dim / 4;
    const int tpb = threads / cpr;
    dim3 grid((d.n_tokens + tpb - 1) / tpb, d.batch);
    rope_kernel<float><<<grid, threads, 0, s>>>((float*)q, (float*)k, d.n_tokens, d.heads,
                                                d.head_dim, d.stride_tok, d.stride_batch, L, tab);
  }
  return cudaGetLastError();
}

}  // namespace mmdit
