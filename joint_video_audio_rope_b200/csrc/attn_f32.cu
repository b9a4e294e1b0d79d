// fp32 attention for fp32 tensors (head_dim 64 or 128): O = softmax(Q K^T
// scale) V per (batch, head) with an online softmax in fp32.
//
// Same operation as the tensor-core path (SkyReels-V4 digest, workflow step 3;
// blog sections 2.1-2.2) for the fp32 dtype, where tensor cores would lose
// precision.  One warp owns one query row; a CTA of 8 warps shares 32-key K/V
// tiles staged in shared memory (K rows padded by one word so that 32 lanes
// reading 32 different keys hit 32 different banks).  Lane i scores key i of
// the tile, so a tile needs one warp max/sum reduction, not one per key.
#include <math.h>

#include "internal.h"

namespace mmdit {

namespace {

constexpr int kRows = 8;   // query rows (warps) per CTA
constexpr int kKeys = 32;  // keys per shared-memory tile

template <int D>
__global__ void __launch_bounds__(kRows * 32) attn_f32_kernel(const F32AttnArgs a) {
  constexpr int C = D / 32;  // channels per lane
  __shared__ float q_s[kRows][D];
  __shared__ float k_s[kKeys][D + 1];
  __shared__ float v_s[kKeys][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y, b = blockIdx.z;
  const int row = blockIdx.x * kRows + warp;
  const bool valid = row < a.Nq;

  const float* qp = a.q + (long long)b * a.q_sb + (long long)row * a.q_st + (long long)h * D;
#pragma unroll
  for (int c = 0; c < C; ++c) q_s[warp][lane + 32 * c] = valid ? qp[lane + 32 * c] : 0.f;

  float m = -INFINITY, l = 0.f, o[C];
#pragma unroll
  for (int c = 0; c < C; ++c) o[c] = 0.f;

  for (int k0 = 0; k0 < a.Nkv; k0 += kKeys) {
    __syncthreads();
    for (int i = threadIdx.x; i < kKeys * D; i += blockDim.x) {
      const int kr = i / D, c = i % D;
      const int key = k0 + kr;
      float kv = 0.f, vv = 0.f;
      if (key < a.Nkv) {
        kv = a.k[(long long)b * a.k_sb + (long long)key * a.k_st + (long long)h * D + c];
        vv = a.v[(long long)b * a.v_sb + (long long)key * a.v_st + (long long)h * D + c];
      }
      k_s[kr][c] = kv;
      v_s[kr][c] = vv;
    }
    __syncthreads();
    const int key = k0 + lane;
    float s = 0.f;
#pragma unroll 8
    for (int c = 0; c < D; ++c) s = fmaf(q_s[warp][c], k_s[lane][c], s);
    s = key < a.Nkv ? s * a.scale : -INFINITY;
    float mt = s;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
    const float mn = fmaxf(m, mt);
    const float p = key < a.Nkv ? expf(s - mn) : 0.f;
    const float corr = (m == -INFINITY) ? 0.f : expf(m - mn);
    float ps = p;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
    l = l * corr + ps;
#pragma unroll
    for (int c = 0; c < C; ++c) o[c] *= corr;
#pragma unroll 4
    for (int jj = 0; jj < kKeys; ++jj) {
      const float pj = __shfl_sync(0xffffffffu, p, jj);
#pragma unroll
      for (int c = 0; c < C; ++c) o[c] = fmaf(pj, v_s[jj][lane + 32 * c], o[c]);
    }
    m = mn;
  }
  if (valid) {
    const float inv = l > 0.f ? 1.f / l : 0.f;
    float* op = a.o + (long long)b * a.o_sb + (long long)row * a.o_st + (long long)h * D;
#pragma unroll
    for (int c = 0; c < C; ++c) op[lane + 32 * c] = o[c] * inv;
    if (a.lse != nullptr && lane == 0)
      a.lse[((long long)b * a.H + h) * a.Nq + row] = l > 0.f ? m + logf(l) : -INFINITY;
  }
}

}  // namespace

cudaError_t launch_attn_f32(const F32AttnArgs& a, cudaStream_t s) {
  if (a.Nq == 0) return cudaSuccess;
  dim3 grid((a.Nq + kRows - 1) / kRows, a.H, a.B);
  if (a.D == 64)
    attn_f32_kernel<64><<<grid, kRows * 32, 0, s>>>(a);
  else
    attn_f32_kernel<128><<<grid, kRows * 32, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace mmdit
