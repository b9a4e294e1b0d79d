// Block-sparse mode, selection side (Prism guide, arXiv 2610.05416, Method
// section 3): key blocks (and, in this library, query blocks too) are
// mean-pooled into representatives; each query block i gets block
// probabilities P_i = softmax_j(Qbar_i . Kbar_j * scale) and attends to
// S_i = TopK(P_i, k) U TopP(P_i, p).
//
// Kernels:
//   pool_kernel    one CTA per (block, batch): each thread sums 8 channels
//                  (one 16-byte vector) of Q and K over the block's <= 64
//                  tokens in fp32 and divides by the real token count.
//                  HBM-bound: Q and K are read once.
//   select_kernel  one CTA per (8 query blocks, head, batch): fp32 block
//                  scores into shared memory, then one warp per row with the
//                  row's probabilities in registers: fp32 probabilities,
//                  fp64 normaliser and prefix masses, value thresholds of the
//                  k-th block (count search) and of the top-p crossing block
//                  (mass search) by bisection on the fp32 bit patterns, and an
//                  ascending-id compaction with warp ballots.  Ranking is P
//                  descending, ties by lower id.
//   groups_kernel  partitions the query blocks into CTA groups of at most the
//                  CTA's query rows and 8 blocks per Q tile (greedy, in block
//                  order).
//   union_kernel   per (group, head, batch): merges the group's selected
//                  lists into one ascending list of 64-row key half-tiles;
//                  an entry holds a start token, a length and a 16-bit
//                  membership mask per 16-token segment (which query blocks
//                  of the group selected that key block).  Consecutive
//                  16-token blocks share an entry.  The attention kernel
//                  walks the list two entries per key tile.
#include <math.h>

#include "internal.h"

namespace mmdit {

namespace {

__global__ void __launch_bounds__(256) pool_kernel(const __nv_bfloat16* __restrict__ q,
                                                   const __nv_bfloat16* __restrict__ k, int H,
                                                   long long st, long long sb, int T, int Hg,
                                                   int Wg, int nblk, float* __restrict__ qbar,
                                                   float* __restrict__ kbar) {
  const int blk = blockIdx.x, b = blockIdx.y;
  int start, len;
  block_extent(T, Hg, Wg, blk, start, len);
  const int nvec = H * 16;  // 16-byte vectors (8 channels) per token row (head_dim 128)
  const float inv = 1.f / (float)len;
  for (int vi = threadIdx.x; vi < nvec; vi += blockDim.x) {
    float aq[8], ak[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) aq[c] = ak[c] = 0.f;
    const long long base = (long long)b * sb + (long long)start * st + 8 * vi;
#pragma unroll 8
    for (int i = 0; i < len; ++i) {
      const uint4 rq = __ldg(reinterpret_cast<const uint4*>(q + base + (long long)i * st));
      const uint4 rk = __ldg(reinterpret_cast<const uint4*>(k + base + (long long)i * st));
      const __nv_bfloat162* pq = reinterpret_cast<const __nv_bfloat162*>(&rq);
      const __nv_bfloat162* pk = reinterpret_cast<const __nv_bfloat162*>(&rk);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float2 fq = __bfloat1622float2(pq[c]), fk = __bfloat1622float2(pk[c]);
        aq[2 * c] += fq.x;
        aq[2 * c + 1] += fq.y;
        ak[2 * c] += fk.x;
        ak[2 * c + 1] += fk.y;
      }
    }
    const int h = vi >> 4, d = (vi & 15) * 8;
    const long long o = (((long long)b * H + h) * nblk + blk) * 128 + d;
    *reinterpret_cast<float4*>(qbar + o) = make_float4(aq[0] * inv, aq[1] * inv, aq[2] * inv, aq[3] * inv);
    *reinterpret_cast<float4*>(qbar + o + 4) = make_float4(aq[4] * inv, aq[5] * inv, aq[6] * inv, aq[7] * inv);
    *reinterpret_cast<float4*>(kbar + o) = make_float4(ak[0] * inv, ak[1] * inv, ak[2] * inv, ak[3] * inv);
    *reinterpret_cast<float4*>(kbar + o + 4) = make_float4(ak[4] * inv, ak[5] * inv, ak[6] * inv, ak[7] * inv);
  }
}

constexpr int kSelRows = 8;
constexpr int kSelChunk = 64;

__device__ __forceinline__ int warp_sum_i(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// One warp holds one row of VPL * 32 probabilities in registers: lane l owns
// blocks l, l + 32, ...; slots past the row hold -1 (a negative bit pattern,
// below every threshold).  Probabilities are >= 0, so their fp32 bit patterns
// order like their values and thresholds are searched on the bits.
template <int VPL>
struct Row {
  float v[VPL];

  // number of probabilities with bit pattern >= tau (tau >= 0)
  __device__ __forceinline__ int count_ge(int tau) const {
    int c = 0;
#pragma unroll
    for (int i = 0; i < VPL; ++i) c += __float_as_int(v[i]) >= tau;
    return warp_sum_i(c);
  }
  // sum of the probabilities with bit pattern >= tau: fp32 over chunks of 8
  // values (each <= 1, error ~1e-7 of the chunk), fp64 across chunks and lanes
  __device__ __forceinline__ double mass_ge(int tau) const {
    double m = 0.0;
#pragma unroll
    for (int i0 = 0; i0 < VPL; i0 += 8) {
      float c = 0.f;
#pragma unroll
      for (int i = i0; i < i0 + 8 && i < VPL; ++i)
        c += __float_as_int(v[i]) >= tau ? v[i] : 0.f;
      m += (double)c;
    }
    return warp_sum_d(m);
  }
};

template <int VPL>
__global__ void __launch_bounds__(256) select_kernel(const float* __restrict__ qbar,
                                                     const float* __restrict__ kbar, int H,
                                                     int nblk, int top_k, float top_p, float scale,
                                                     int cap, int32_t* __restrict__ idx,
                                                     int32_t* __restrict__ cnt) {
  extern __shared__ float sm[];
  float* q_s = sm;                                  // [8][128]
  float* k_s = q_s + kSelRows * 128;                // [64][129]
  float* sc = k_s + kSelChunk * 129;                // [8][nblk]
  const int h = blockIdx.y, b = blockIdx.z;
  const int r0 = blockIdx.x * kSelRows;
  const long long hb = ((long long)b * H + h) * nblk;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  for (int i = tid; i < kSelRows * 128; i += 256) {
    const int r = i >> 7;
    q_s[i] = (r0 + r < nblk) ? qbar[(hb + r0 + r) * 128 + (i & 127)] : 0.f;
  }
  // ---- scores: sc[r][j] = qbar_r . kbar_j * scale (fp32)
  for (int c0 = 0; c0 < nblk; c0 += kSelChunk) {
    __syncthreads();
    for (int i = tid; i < kSelChunk * 128; i += 256) {
      const int kr = i >> 7, c = i & 127;
      k_s[kr * 129 + c] = (c0 + kr < nblk) ? kbar[(hb + c0 + kr) * 128 + c] : 0.f;
    }
    __syncthreads();
    const int kk = tid & 63, ra = tid >> 6, rb = ra + 4;
    float da = 0.f, db = 0.f;
#pragma unroll 16
    for (int c = 0; c < 128; ++c) {
      const float kv = k_s[kk * 129 + c];
      da = fmaf(q_s[ra * 128 + c], kv, da);
      db = fmaf(q_s[rb * 128 + c], kv, db);
    }
    if (c0 + kk < nblk) {
      sc[ra * nblk + c0 + kk] = da * scale;
      sc[rb * nblk + c0 + kk] = db * scale;
    }
  }
  __syncthreads();

  // ---- per row selection: one warp per query block, the row in registers
  const int row = r0 + warp;
  if (row >= nblk) return;
  const int n = nblk;
  const float* srow = sc + warp * nblk;
  Row<VPL> P;
  float mx = -INFINITY;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int j = lane + 32 * i;
    P.v[i] = j < n ? srow[j] : -INFINITY;
    mx = fmaxf(mx, P.v[i]);
  }
  mx = warp_max_f(mx);
  double z = 0.0;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int j = lane + 32 * i;
    // unnormalised probability in (0, 1]; -1 marks the slots past the row
    P.v[i] = j < n ? expf(P.v[i] - mx) : -1.f;
    if (j < n) z += (double)P.v[i];
  }
  z = warp_sum_d(z);

  const int kOne = 0x3F800000;  // bit pattern of 1.0f, the largest value
  // top-k threshold: largest tau with count(P >= tau) >= k'
  const int kq = min(max(top_k, 0), n);
  int tau_k = kOne + 1;  // nothing selected by top-k when k' == 0
  if (kq > 0) {
    int lo = 0, hi = kOne + 1;
    while (hi - lo > 1) {
      const int mid = lo + ((hi - lo) >> 1);
      if (P.count_ge(mid) >= kq) lo = mid; else hi = mid;
    }
    tau_k = lo;
  }
  // top-p threshold: largest tau with mass(P >= tau) >= p * Z
  const double target = (double)top_p * z;
  const double mass_all = P.mass_ge(0);
  int tau_p;
  if (target <= 0.0) {
    tau_p = kOne;
  } else if (mass_all < target) {
    tau_p = 0;  // the sum never reaches p (p >= 1 with rounding): all blocks
  } else {
    int lo = 0, hi = kOne + 1;
    while (hi - lo > 1) {
      const int mid = lo + ((hi - lo) >> 1);
      if (P.mass_ge(mid) >= target) lo = mid; else hi = mid;
    }
    tau_p = lo;
  }
  int take_p;  // how many blocks top-p selects
  {
    const int c_gt = P.count_ge(tau_p + 1);
    const int c_eq = P.count_ge(tau_p) - c_gt;
    const double m_gt = P.mass_ge(tau_p + 1);
    const double tv = (double)__int_as_float(tau_p);
    int m = 1;
    if (tau_p == 0 && target > 0.0 && mass_all < target) {
      m = c_eq;  // everything
    } else if (target > m_gt && tv > 0.0) {
      m = (int)ceil((target - m_gt) / tv);
    }
    m = c_eq > 0 ? max(1, min(m, c_eq)) : 0;
    take_p = c_gt + m;
  }
  // final threshold and number of tied blocks to take (lowest ids first)
  int tau, take_eq;
  if (take_p >= kq) {
    tau = tau_p;
    take_eq = take_p - P.count_ge(tau_p + 1);
  } else {
    tau = tau_k;
    take_eq = kq - P.count_ge(tau_k + 1);
  }
  // ---- ascending compaction
  int32_t* out = idx + (hb + row) * (long long)cap;
  int pos = 0, ties = 0;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int j = lane + 32 * i;
    const int vb = __float_as_int(P.v[i]);
    const bool eq = vb == tau;  // padding (-1) never equals tau >= 0
    const unsigned eqm = __ballot_sync(0xffffffffu, eq);
    const int tie_rank = ties + __popc(eqm & ((1u << lane) - 1u));
    const bool sel = vb > tau || (eq && tie_rank < take_eq);
    const unsigned sm_ = __ballot_sync(0xffffffffu, sel);
    if (sel) out[pos + __popc(sm_ & ((1u << lane) - 1u))] = j;
    pos += __popc(sm_);
    ties += __popc(eqm);
  }
  if (lane == 0) cnt[hb + row] = pos;
}

// Greedy partition of the query blocks into groups of <= kGroupTokens tokens
// and <= kGroupBlocks blocks; must agree with the host-side count
// (mmdit_api.cu).
__global__ void groups_kernel(int T, int H, int W, int nblk, int4* groups) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  int g = 0, first = 0, nb = 0, tokens = 0, start = 0;
  for (int b = 0; b < nblk; ++b) {
    int st, len;
    block_extent(T, H, W, b, st, len);
    if (nb == kGroupBlocks || tokens + len > kGroupTokens) {
      groups[g++] = make_int4(first, nb, start, tokens);
      first = b;
      nb = 0;
      tokens = 0;
      start = st;
    }
    if (nb == 0) start = st;
    ++nb;
    tokens += len;
  }
  if (nb > 0) groups[g++] = make_int4(first, nb, start, tokens);
}

// Block-wide inclusive scans over one value per thread (256 threads).
__device__ __forceinline__ int block_scan_sum(int v, int* wsum, int lane, int warp, int& total) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) wsum[warp] = v;
  __syncthreads();
  int before = 0;
  total = 0;
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    before += (w < warp) ? wsum[w] : 0;
    total += wsum[w];
  }
  __syncthreads();
  return v + before;
}
__device__ __forceinline__ int block_scan_max(int v, int* wmax, int lane, int warp) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v = max(v, n);
  }
  if (lane == 31) wmax[warp] = v;
  __syncthreads();
  int before = -1;
#pragma unroll
  for (int w = 0; w < 8; ++w) before = (w < warp) ? max(before, wmax[w]) : before;
  __syncthreads();
  return max(v, before);
}

// Merged key-block list of one query group.  Entry = one 64-row half of an
// attention key tile: {start token, length, membership masks of its four
// 16-token segments (16 bits each: which query blocks of the group selected
// the key block the segment belongs to)}.  A 64-token block is one entry;
// runs of consecutive 16-token blocks (the short last t-slab), which are
// contiguous in block-major storage, are packed four to an entry.
__global__ void __launch_bounds__(256) union_kernel(const int32_t* __restrict__ idx,
                                                    const int32_t* __restrict__ cnt, int cap,
                                                    const int4* __restrict__ groups, int H,
                                                    int nblk, int n_groups, int T, int Hg, int Wg,
                                                    uint4* __restrict__ ulist,
                                                    int* __restrict__ ucnt) {
  extern __shared__ uint32_t mask[];  // [nblk]
  __shared__ int wtmp[8];
  const int g = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int4 gr = groups[g];
  for (int j = tid; j < nblk; j += 256) mask[j] = 0u;
  __syncthreads();
  const long long hb = ((long long)b * H + h) * nblk;
  for (int i = 0; i < gr.y; ++i) {
    const long long r = hb + gr.x + i;
    const int c = min(max(cnt[r], 0), nblk);
    for (int e = tid; e < c; e += 256) {
      const int j = idx[r * cap + e];
      if ((unsigned)j < (unsigned)nblk) atomicOr(&mask[j], 1u << i);
    }
  }
  __syncthreads();
  const long long lid = ((long long)b * H + h) * n_groups + g;
  uint4* out = ulist + lid * nblk;
  auto packable = [&](int j) {
    if (j < 0 || j >= nblk || mask[j] == 0u) return false;
    int st, len;
    block_extent(T, Hg, Wg, j, st, len);
    return len == 16;
  };
  int running = 0, run_carry = -1;
  for (int j0 = 0; j0 < nblk; j0 += 256) {
    const int j = j0 + tid;
    const bool in = j < nblk && mask[j] != 0u;
    const bool pk = in && packable(j);
    // start of a run of consecutive packable blocks
    const bool run_start = pk && !packable(j - 1);
    int last_start = block_scan_max(run_start ? j : -1, wtmp, lane, warp);
    last_start = max(last_start, run_carry);
    const int rank = pk ? j - last_start : 0;
    const bool leader = in && (!pk || (rank & 3) == 0);
    int total;
    const int pos = block_scan_sum(leader ? 1 : 0, wtmp, lane, warp, total) - (leader ? 1 : 0);
    if (leader) {
      int st, len;
      block_extent(T, Hg, Wg, j, st, len);
      uint32_t m[4];
      if (!pk) {
        m[0] = m[1] = m[2] = m[3] = mask[j];
      } else {
        m[0] = mask[j];
        len = 16;
        m[1] = m[2] = m[3] = 0u;
        for (int q = 1; q < 4 && packable(j + q); ++q) {
          m[q] = mask[j + q];
          len += 16;
        }
      }
      out[running + pos] = make_uint4((uint32_t)st, (uint32_t)len, m[0] | (m[1] << 16),
                                      m[2] | (m[3] << 16));
    }
    running += total;
    // the last thread's run start carries into the next chunk
    if (tid == 255) wtmp[0] = last_start;
    __syncthreads();
    run_carry = wtmp[0];
    __syncthreads();
  }
  if (tid == 0) ucnt[lid] = running;
}

}  // namespace

size_t select_smem_bytes(int nblk) {
  return sizeof(float) * ((size_t)kSelRows * 128 + (size_t)kSelChunk * 129 + (size_t)kSelRows * nblk);
}

cudaError_t launch_pool(const __nv_bfloat16* q, const __nv_bfloat16* k, const mmdit_tensor_desc& d,
                        int T, int H, int W, int nblk, float* qbar, float* kbar, cudaStream_t s) {
  if (nblk == 0) return cudaSuccess;
  pool_kernel<<<dim3(nblk, d.batch), 256, 0, s>>>(q, k, d.heads, d.stride_tok, d.stride_batch, T,
                                                  H, W, nblk, qbar, kbar);
  return cudaGetLastError();
}

template <int VPL>
cudaError_t launch_select_vpl(const float* qbar, const float* kbar, int B, int H, int nblk,
                              int top_k, float top_p, float scale, int cap, int32_t* idx,
                              int32_t* cnt, cudaStream_t s) {
  const size_t smem = select_smem_bytes(nblk);
  // the attribute is raised to the largest size this library uses, once per device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess)
    e = once_per_device(dev, [] {
      return cudaFuncSetAttribute(select_kernel<VPL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)select_smem_bytes(kMaxBlocks));
    });
  if (e != cudaSuccess) return e;
  dim3 grid((nblk + kSelRows - 1) / kSelRows, H, B);
  select_kernel<VPL><<<grid, 256, smem, s>>>(qbar, kbar, H, nblk, top_k, top_p, scale, cap, idx,
                                             cnt);
  return cudaGetLastError();
}

cudaError_t launch_select(const float* qbar, const float* kbar, int B, int H, int nblk, int top_k,
                          float top_p, float scale, int cap, int32_t* idx, int32_t* cnt,
                          cudaStream_t s) {
  if (nblk == 0) return cudaSuccess;
  // registers per lane: the row rounded up to a multiple of 32 x {8, 32, 64, 96, 128, 192}
  const int vpl = (nblk + 31) / 32;
#define MMDIT_SEL(V) \
  if (vpl <= V) return launch_select_vpl<V>(qbar, kbar, B, H, nblk, top_k, top_p, scale, cap, idx, cnt, s)
  MMDIT_SEL(8);
  MMDIT_SEL(32);
  MMDIT_SEL(64);
  MMDIT_SEL(96);
  MMDIT_SEL(128);
  MMDIT_SEL(192);
#undef MMDIT_SEL
  return cudaErrorInvalidValue;  // more blocks than the library supports (checked earlier)
}

cudaError_t launch_groups(int T, int H, int W, int nblk, int4* groups, int*, cudaStream_t s) {
  groups_kernel<<<1, 32, 0, s>>>(T, H, W, nblk, groups);
  return cudaGetLastError();
}

cudaError_t launch_union(const int32_t* idx, const int32_t* cnt, int cap, const int4* groups,
                         int n_groups, const int*, int B, int H, int nblk, int T, int Hg,
                         int Wg, uint4* ulist, int* ucnt, cudaStream_t s) {
  if (n_groups == 0) return cudaSuccess;
  const size_t smem = sizeof(uint32_t) * (size_t)nblk;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess)
    e = once_per_device(dev, [] {
      return cudaFuncSetAttribute(union_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)(sizeof(uint32_t) * kMaxBlocks));
    });
  if (e != cudaSuccess) return e;
  union_kernel<<<dim3(n_groups, H, B), 256, smem, s>>>(idx, cnt, cap, groups, H, nblk, n_groups,
                                                       T, Hg, Wg, ulist, ucnt);
  return cudaGetLastError();
}

}  // namespace mmdit
