// Block-sparse mode, selection side (Prism guide, arXiv 2610.05416, Method
// section 3): key blocks (and, in this library, query blocks too) are
// mean-pooled into representatives; each query block i gets block
// probabilities P_i = softmax_j(Qbar_i . Kbar_j * scale) and attends to
// S_i = TopK(P_i, k) U TopP(P_i, p).
//
// Every kernel reads the block geometry from a block table: per batch item,
// {start token, length} of each block in storage order plus the block count.
// The fixed 4x4x4 mode fills the table from the grid (grid_table_kernel); the
// content-adaptive mode (Prism guide, Method sections 1-2; prism.cu) writes
// it from its per-zone plan.  Blocks hold 1..256 tokens.
//
// Kernels:
//   grid_table_kernel  the table of the 4x4x4 blocks of a block-major grid.
//   pool_kernel        one CTA per (block, 128 16-byte vectors, batch): each
//                      thread sums one vector (8 channels of one head) of Q
//                      and K over the block's tokens in fp32 and divides by
//                      the token count.  HBM-bound: Q and K are read once.
//   scores_kernel      S = Qbar Kbar^T * scale per (batch, head): fp32 SGEMM
//                      on the CUDA cores (the selection decision is taken in
//                      fp32), 128 x 128 tiles, 8 x 8 outputs per thread,
//                      16-channel double-buffered shared-memory stages.
//   select_rows_kernel one warp per (row, head, batch), the row's scores in
//                      registers: fp32 probabilities, fp64 normaliser and
//                      prefix masses, the value threshold of the top-p
//                      crossing block (mass search) and, only when top-p
//                      takes fewer than k blocks, of the k-th block (count
//                      search), both by bisection on the fp32 bit patterns;
//                      ascending-id compaction with warp ballots.  Ranking
//                      is P descending, ties by lower id.
//   groups_kernel      partitions the query blocks into CTA groups of at
//                      most the CTA's query rows and 8 blocks per Q tile
//                      (greedy, in block order).
//   union_kernel       per (group, head, batch): merges the group's selected
//                      lists into one ascending list of key entries of <= 64
//                      rows; an entry holds a start token, a length and a
//                      16-bit membership mask per 16-token segment (which
//                      query blocks of the group selected that key block).
//                      A block of L tokens gives ceil(L / 64) entries; runs of
//                      consecutive 16-token blocks share an entry.  The
//                      attention kernel walks the list two entries per key
//                      tile.
//   schedule_kernel    lists the (group, head, batch) items whose group
//                      exists, in index order, for the sparse attention
//                      launch (CTA i takes the i-th listed item).
#include <math.h>

#include "internal.h"

namespace mmdit {

namespace {

// ------------------------------------------------------------------ tables

__global__ void grid_table_kernel(int T, int H, int W, int nblk, int maxb, int2* __restrict__ tab,
                                  int* __restrict__ tab_n) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  const int b = blockIdx.y;
  if (j < nblk) {
    int st, len;
    block_extent(T, H, W, j, st, len);
    tab[(long long)b * maxb + j] = make_int2(st, len);
  }
  if (j == 0) tab_n[b] = nblk;
}

// Block j of batch item b with its entry checked against the sequence: an
// entry outside [0, N) or longer than kMaxBlockTokens is treated as empty
// (and recorded in the error word by builds with device-side checks).
__device__ __forceinline__ int2 table_entry(const int2* tab, int maxb, int b, int j, int N,
                                            int* err) {
  int2 e = tab[(long long)b * maxb + j];
  const bool ok = e.x >= 0 && e.y >= 0 && e.y <= kMaxBlockTokens && e.x <= N - e.y;
  MMDIT_DCHECK(ok, err);
  if (!ok) e = make_int2(0, 0);
  return e;
}

// Block count of batch item b, clamped to the table's capacity.
__device__ __forceinline__ int table_count(const int* tab_n, int b, int maxb, int* err) {
  const int n = tab_n[b];
  MMDIT_DCHECK(n >= 0 && n <= maxb, err);
  return min(max(n, 0), maxb);
}

// ------------------------------------------------------------------ pooling

constexpr int kPoolThreads = 128;

__global__ void __launch_bounds__(kPoolThreads) pool_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k, int H, int N,
    long long st, long long sb, const int2* __restrict__ tab, const int* __restrict__ tab_n,
    int maxb, float* __restrict__ qbar, float* __restrict__ kbar, int* err) {
  const int blk = blockIdx.x, b = blockIdx.z;
  const int vi = blockIdx.y * kPoolThreads + threadIdx.x;  // 16-byte vector of the token row
  if (blk >= table_count(tab_n, b, maxb, err) || vi >= H * 16) return;
  const int2 e = table_entry(tab, maxb, b, blk, N, err);
  float aq[8], ak[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) aq[c] = ak[c] = 0.f;
  const __nv_bfloat16* pq0 = q + (long long)b * sb + (long long)e.x * st + 8 * vi;
  const __nv_bfloat16* pk0 = k + (long long)b * sb + (long long)e.x * st + 8 * vi;
#pragma unroll 8
  for (int i = 0; i < e.y; ++i) {
    const uint4 rq = __ldg(reinterpret_cast<const uint4*>(pq0 + (long long)i * st));
    const uint4 rk = __ldg(reinterpret_cast<const uint4*>(pk0 + (long long)i * st));
    const __nv_bfloat162* hq = reinterpret_cast<const __nv_bfloat162*>(&rq);
    const __nv_bfloat162* hk = reinterpret_cast<const __nv_bfloat162*>(&rk);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const float2 fq = __bfloat1622float2(hq[c]), fk = __bfloat1622float2(hk[c]);
      aq[2 * c] += fq.x;
      aq[2 * c + 1] += fq.y;
      ak[2 * c] += fk.x;
      ak[2 * c + 1] += fk.y;
    }
  }
  const float inv = e.y > 0 ? 1.f / (float)e.y : 0.f;
  const int h = vi >> 4, d = (vi & 15) * 8;
  const long long o = (((long long)b * H + h) * maxb + blk) * 128 + d;
  *reinterpret_cast<float4*>(qbar + o) = make_float4(aq[0] * inv, aq[1] * inv, aq[2] * inv, aq[3] * inv);
  *reinterpret_cast<float4*>(qbar + o + 4) = make_float4(aq[4] * inv, aq[5] * inv, aq[6] * inv, aq[7] * inv);
  *reinterpret_cast<float4*>(kbar + o) = make_float4(ak[0] * inv, ak[1] * inv, ak[2] * inv, ak[3] * inv);
  *reinterpret_cast<float4*>(kbar + o + 4) = make_float4(ak[4] * inv, ak[5] * inv, ak[6] * inv, ak[7] * inv);
}

// ------------------------------------------------------------------ scores

constexpr int kSgTile = 128;  // output tile edge
constexpr int kSgK = 16;      // channels per shared-memory stage
constexpr int kSgPad = kSgTile + 4;

// S[b][h][i][j] = scale * sum_c qbar[b][h][i][c] kbar[b][h][j][c] for i, j
// below the batch item's block count; rows of S are `ld` floats apart.
// Thread (tx, ty) of the 16 x 16 grid owns rows {4ty..4ty+3, 64+4ty..64+4ty+3}
// and columns {4tx..4tx+3, 64+4tx..64+4tx+3} of the tile: per channel two
// float4 loads of each operand feed 64 FMAs.  The operands are stored
// channel-major in shared memory (transposed on the way in).
__global__ void __launch_bounds__(256, 2) scores_kernel(const float* __restrict__ qbar,
                                                     const float* __restrict__ kbar,
                                                     const int* __restrict__ tab_n, int H,
                                                     int maxb, int ld, float scale,
                                                     float* __restrict__ S, int* err) {
  __shared__ __align__(16) float As[2][kSgK][kSgPad];
  __shared__ __align__(16) float Bs[2][kSgK][kSgPad];
  const int bh = blockIdx.z, b = bh / H;
  const int n = table_count(tab_n, b, maxb, err);
  const int m0 = blockIdx.y * kSgTile, n0 = blockIdx.x * kSgTile;
  if (m0 >= n || n0 >= n) return;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const float* A = qbar + (long long)bh * maxb * 128;
  const float* Bm = kbar + (long long)bh * maxb * 128;
  // loader: 512 float4 per operand stage, two per thread (row, 4-channel group)
  float4 ra[2], rb[2];
  auto load = [&](int k0) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int idx = tid + 256 * i, row = idx >> 2, c4 = idx & 3;
      const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
      ra[i] = (m0 + row < n) ? *reinterpret_cast<const float4*>(A + (long long)(m0 + row) * 128 + k0 + 4 * c4) : z;
      rb[i] = (n0 + row < n) ? *reinterpret_cast<const float4*>(Bm + (long long)(n0 + row) * 128 + k0 + 4 * c4) : z;
    }
  };
  auto store = [&](int buf) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int idx = tid + 256 * i, row = idx >> 2, c4 = idx & 3;
      As[buf][4 * c4 + 0][row] = ra[i].x;
      As[buf][4 * c4 + 1][row] = ra[i].y;
      As[buf][4 * c4 + 2][row] = ra[i].z;
      As[buf][4 * c4 + 3][row] = ra[i].w;
      Bs[buf][4 * c4 + 0][row] = rb[i].x;
      Bs[buf][4 * c4 + 1][row] = rb[i].y;
      Bs[buf][4 * c4 + 2][row] = rb[i].z;
      Bs[buf][4 * c4 + 3][row] = rb[i].w;
    }
  };
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  load(0);
  store(0);
  __syncthreads();
#pragma unroll 1
  for (int s = 0; s < 128 / kSgK; ++s) {
    const int buf = s & 1;
    if (s + 1 < 128 / kSgK) load((s + 1) * kSgK);
#pragma unroll
    for (int kk = 0; kk < kSgK; ++kk) {
      const float4 a0 = *reinterpret_cast<const float4*>(&As[buf][kk][4 * ty]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[buf][kk][64 + 4 * ty]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[buf][kk][4 * tx]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[buf][kk][64 + 4 * tx]);
      const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], bv[j], acc[i][j]);
    }
    if (s + 1 < 128 / kSgK) store(buf ^ 1);
    __syncthreads();
  }
  float* Sbh = S + (long long)bh * maxb * ld;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int row = m0 + (i < 4 ? 4 * ty + i : 64 + 4 * ty + i - 4);
    if (row >= maxb) continue;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int col = n0 + half * 64 + 4 * tx;
      if (col >= ld) continue;
      *reinterpret_cast<float4*>(Sbh + (long long)row * ld + col) =
          make_float4(acc[i][4 * half] * scale, acc[i][4 * half + 1] * scale,
                      acc[i][4 * half + 2] * scale, acc[i][4 * half + 3] * scale);
    }
  }
}

// ------------------------------------------------------------------ selection

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
  // values per lane that hold blocks of the row (the rest are padding, -1):
  // the passes skip the chunks of 8 past them (warp-uniform branches), so a
  // row of n blocks costs ~n, not the capacity the template was sized for
  int nv = VPL;

  // number of probabilities with bit pattern >= tau (tau >= 0)
  __device__ __forceinline__ int count_ge(int tau) const {
    int c = 0;
#pragma unroll
    for (int i0 = 0; i0 < VPL; i0 += 8) {
      if (i0 < nv) {  // warp-uniform
#pragma unroll
        for (int i = i0; i < i0 + 8 && i < VPL; ++i) c += __float_as_int(v[i]) >= tau;
      }
    }
    return warp_sum_i(c);
  }
  // sum of the probabilities with bit pattern >= tau: fp32 over chunks of 8
  // values (each <= 1, error ~1e-7 of the chunk), fp64 across chunks and lanes
  __device__ __forceinline__ double mass_ge(int tau) const {
    double m = 0.0;
#pragma unroll
    for (int i0 = 0; i0 < VPL; i0 += 8) {
      if (i0 < nv) {  // warp-uniform
        float c = 0.f;
#pragma unroll
        for (int i = i0; i < i0 + 8 && i < VPL; ++i)
          c += __float_as_int(v[i]) >= tau ? v[i] : 0.f;
        m += (double)c;
      }
    }
    return warp_sum_d(m);
  }
};

template <int VPL>
__global__ void __launch_bounds__(256) select_rows_kernel(
    const float* __restrict__ S, const int* __restrict__ tab_n, int H, int maxb, int ld,
    int top_k, float top_p, int cap, int32_t* __restrict__ idx, int32_t* __restrict__ cnt,
    int* err) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y, b = blockIdx.z;
  const int row = blockIdx.x * 8 + warp;
  const int n = table_count(tab_n, b, maxb, err);
  if (row >= n) return;
  const long long hb = ((long long)b * H + h) * maxb;
  const float* srow = S + (hb + row) * ld;
  Row<VPL> P;
  P.nv = (n + 31) / 32;
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
  const int cp_gt = P.count_ge(tau_p + 1);
  {
    const int c_eq = P.count_ge(tau_p) - cp_gt;
    const double m_gt = P.mass_ge(tau_p + 1);
    const double tv = (double)__int_as_float(tau_p);
    int m = 1;
    if (tau_p == 0 && target > 0.0 && mass_all < target) {
      m = c_eq;  // everything
    } else if (target > m_gt && tv > 0.0) {
      m = (int)ceil((target - m_gt) / tv);
    }
    m = c_eq > 0 ? max(1, min(m, c_eq)) : 0;
    take_p = cp_gt + m;
  }
  // top-k only matters when top-p takes fewer than k' blocks
  const int kq = min(max(top_k, 0), n);
  int tau, take_eq;
  if (take_p >= kq) {
    tau = tau_p;
    take_eq = take_p - cp_gt;
  } else {
    // largest tau with count(P >= tau) >= k'
    int lo = 0, hi = kOne + 1;
    while (hi - lo > 1) {
      const int mid = lo + ((hi - lo) >> 1);
      if (P.count_ge(mid) >= kq) lo = mid; else hi = mid;
    }
    tau = lo;
    take_eq = kq - P.count_ge(lo + 1);
  }
  // ---- ascending compaction
  int32_t* out = idx + (hb + row) * (long long)cap;
  int pos = 0, ties = 0;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    if (i < P.nv) {  // only padding beyond (warp-uniform)
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
  }
  if (lane == 0) cnt[hb + row] = pos;
}

// ------------------------------------------------------------------ groups

// Greedy partition of each batch item's query blocks, in block order, into
// groups of <= kGroupTokens tokens and <= kGroupBlocks blocks: {first block,
// blocks, start token, tokens}.  One warp per batch item: the lanes fetch 32
// table entries at a time and every lane runs the same greedy walk over them
// (shuffled), lane 0 writing the groups.
__global__ void groups_kernel(const int2* __restrict__ tab, const int* __restrict__ tab_n,
                              int maxb, int N, int maxg, int4* __restrict__ groups,
                              int* __restrict__ n_groups, int* err) {
  const int b = blockIdx.x, lane = threadIdx.x;
  const int n = table_count(tab_n, b, maxb, err);
  int g = 0, first = 0, nb = 0, tokens = 0, start = 0;
  int4* out = groups + (long long)b * maxg;
  for (int j0 = 0; j0 < n; j0 += 32) {
    const int2 mine = (j0 + lane < n) ? table_entry(tab, maxb, b, j0 + lane, N, err)
                                      : make_int2(0, 0);
    const int m = min(32, n - j0);
    for (int i = 0; i < m; ++i) {
      const int st = __shfl_sync(0xffffffffu, mine.x, i);
      const int len = __shfl_sync(0xffffffffu, mine.y, i);
      if (nb == kGroupBlocks || tokens + len > kGroupTokens) {
        MMDIT_DCHECK(g < maxg, err);
        if (lane == 0 && g < maxg) out[g] = make_int4(first, nb, start, tokens);
        ++g;
        first = j0 + i;
        nb = 0;
        tokens = 0;
      }
      if (nb == 0) start = st;
      ++nb;
      tokens += len;
    }
  }
  if (nb > 0) {
    if (lane == 0 && g < maxg) out[g] = make_int4(first, nb, start, tokens);
    ++g;
  }
  if (lane == 0) n_groups[b] = min(g, maxg);
}

// ------------------------------------------------------------------ union

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

// Merged key list of one query group (see the file comment).  Entries past
// `ucap` are never written (the capacity bounds every list by construction;
// device-checked builds record a violation).
__global__ void __launch_bounds__(256) union_kernel(
    const int32_t* __restrict__ idx, const int32_t* __restrict__ cnt, int cap,
    const int2* __restrict__ tab, const int* __restrict__ tab_n, int maxb, int N,
    const int4* __restrict__ groups, const int* __restrict__ n_groups, int maxg, int H,
    int ucap, uint4* __restrict__ ulist, int* __restrict__ ucnt, int* err) {
  extern __shared__ uint32_t mask[];  // [maxb]
  __shared__ int wtmp[8];
  const int g = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long lid = ((long long)b * H + h) * maxg + g;
  const int ng = min(max(n_groups[b], 0), maxg);
  if (g >= ng) {
    if (tid == 0) ucnt[lid] = 0;
    return;
  }
  const int n = table_count(tab_n, b, maxb, err);
  const int4 gr = groups[(long long)b * maxg + g];
  for (int j = tid; j < n; j += 256) mask[j] = 0u;
  __syncthreads();
  const long long hb = ((long long)b * H + h) * maxb;
  for (int i = 0; i < gr.y; ++i) {
    const long long r = hb + gr.x + i;
    const int c0 = cnt[r];
    MMDIT_DCHECK(c0 >= 0 && c0 <= n, err);
    const int c = min(max(c0, 0), n);
    for (int e = tid; e < c; e += 256) {
      const int j = idx[r * cap + e];
      MMDIT_DCHECK((unsigned)j < (unsigned)n, err);
      if ((unsigned)j < (unsigned)n) atomicOr(&mask[j], 1u << i);
    }
#ifdef MMDIT_DEVICE_CHECKS
    // the list must be strictly ascending
    for (int e = tid + 1; e < c; e += 256) MMDIT_DCHECK(idx[r * cap + e - 1] < idx[r * cap + e], err);
#endif
  }
  __syncthreads();
  uint4* out = ulist + lid * ucap;
  auto len_of = [&](int j) { return table_entry(tab, maxb, b, j, N, err).y; };
  auto packable = [&](int j) { return j >= 0 && j < n && mask[j] != 0u && len_of(j) == 16; };
  int running = 0, run_carry = -1;
  for (int j0 = 0; j0 < n; j0 += 256) {
    const int j = j0 + tid;
    const bool in = j < n && mask[j] != 0u;
    const int2 ent = in ? table_entry(tab, maxb, b, j, N, err) : make_int2(0, 0);
    const bool pk = in && ent.y == 16;
    // start of a run of consecutive packable blocks
    const bool run_start = pk && !packable(j - 1);
    int last_start = block_scan_max(run_start ? j : -1, wtmp, lane, warp);
    last_start = max(last_start, run_carry);
    const int rank = pk ? j - last_start : 0;
    // entries this block starts: a packed run starts one every four blocks;
    // any other selected block gives one entry per 64 rows
    const int n_ent = !in ? 0 : (pk ? ((rank & 3) == 0 ? 1 : 0) : (ent.y + 63) / 64);
    int total;
    const int pos = block_scan_sum(n_ent, wtmp, lane, warp, total) - n_ent;
    if (n_ent > 0) {
      if (pk) {
        uint32_t m[4] = {mask[j], 0u, 0u, 0u};
        int len = 16;
        for (int qq = 1; qq < 4 && packable(j + qq); ++qq) {
          m[qq] = mask[j + qq];
          len += 16;
        }
        if (running + pos < ucap)
          out[running + pos] = make_uint4((uint32_t)ent.x, (uint32_t)len, m[0] | (m[1] << 16),
                                          m[2] | (m[3] << 16));
      } else {
        const uint32_t mm = mask[j] | (mask[j] << 16);
        for (int e = 0; e < n_ent; ++e)
          if (running + pos + e < ucap)
            out[running + pos + e] = make_uint4((uint32_t)(ent.x + 64 * e),
                                                (uint32_t)min(64, ent.y - 64 * e), mm, mm);
      }
    }
    running += total;
    // the last thread's run start carries into the next chunk
    if (tid == 255) wtmp[0] = last_start;
    __syncthreads();
    run_carry = wtmp[0];
    __syncthreads();
  }
  MMDIT_DCHECK(running <= ucap, err);
  if (tid == 0) ucnt[lid] = min(running, ucap);
}

// ------------------------------------------------------------------ schedule

constexpr int kSchedThreads = 1024;

// The work items of the sparse attention: every (group, head, batch) item
// whose group exists, in index order (batch, head, group) --
// consecutive items are neighbouring query groups of one head, which select
// largely the same key blocks, so the CTAs running side by side share their
// K/V tiles through L2.  (Ordering by list length, longest first, measured
// 10 % slower on the 1080p layer: it scattered the concurrent items over the
// heads.)  order[0 .. *n_order) lists item ids (b H + h) maxg + g.
__global__ void __launch_bounds__(kSchedThreads) schedule_kernel(
    const int* __restrict__ n_groups, int maxg, int H, int n_items, int* __restrict__ order,
    int* __restrict__ n_order) {
  __shared__ int wsum[kSchedThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (n_items + kSchedThreads - 1) / kSchedThreads;
  const int lo = min(n_items, tid * per), hi = min(n_items, lo + per);
  auto real = [&](int it) { return it % maxg < n_groups[it / (maxg * H)]; };
  int c = 0;
  for (int it = lo; it < hi; ++it) c += real(it);
  int x = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += t;
  }
  if (lane == 31) wsum[warp] = x;
  __syncthreads();
  int before = 0, total = 0;
  for (int w = 0; w < kSchedThreads / 32; ++w) {
    before += w < warp ? wsum[w] : 0;
    total += wsum[w];
  }
  int pos = before + x - c;
  for (int it = lo; it < hi; ++it)
    if (real(it)) order[pos++] = it;
  if (tid == 0) *n_order = total;
}

}  // namespace

// ---------------------------------------------------------------------- host

cudaError_t launch_grid_table(int T, int H, int W, int nblk, int B, int maxb, int2* tab,
                              int* tab_n, cudaStream_t s) {
  grid_table_kernel<<<dim3((nblk + 255) / 256 + (nblk == 0), B), 256, 0, s>>>(T, H, W, nblk,
                                                                              maxb, tab, tab_n);
  return cudaGetLastError();
}

size_t select_scores_ld(int maxb) { return (size_t)((maxb + 3) / 4) * 4; }

cudaError_t launch_pool(const __nv_bfloat16* q, const __nv_bfloat16* k, const mmdit_tensor_desc& d,
                        const int2* tab, const int* tab_n, int maxb, float* qbar, float* kbar,
                        int* err, cudaStream_t s) {
  if (maxb == 0) return cudaSuccess;
  dim3 grid(maxb, (d.heads * 16 + kPoolThreads - 1) / kPoolThreads, d.batch);
  pool_kernel<<<grid, kPoolThreads, 0, s>>>(q, k, d.heads, d.n_tokens, d.stride_tok,
                                            d.stride_batch, tab, tab_n, maxb, qbar, kbar, err);
  return cudaGetLastError();
}

template <int VPL>
cudaError_t launch_select_vpl(const float* S, const int* tab_n, int B, int H, int maxb, int top_k,
                              float top_p, int cap, int32_t* idx, int32_t* cnt, int* err,
                              cudaStream_t s) {
  dim3 grid((maxb + 7) / 8, H, B);
  select_rows_kernel<VPL><<<grid, 256, 0, s>>>(S, tab_n, H, maxb, (int)select_scores_ld(maxb),
                                               top_k, top_p, cap, idx, cnt, err);
  return cudaGetLastError();
}

cudaError_t launch_select(const float* qbar, const float* kbar, const int* tab_n, int B, int H,
                          int maxb, int top_k, float top_p, float scale, int cap, float* S,
                          int32_t* idx, int32_t* cnt, int* err, cudaStream_t s) {
  if (maxb == 0) return cudaSuccess;
  const int tiles = (maxb + kSgTile - 1) / kSgTile;
  scores_kernel<<<dim3(tiles, tiles, B * H), 256, 0, s>>>(qbar, kbar, tab_n, H, maxb,
                                                          (int)select_scores_ld(maxb), scale, S,
                                                          err);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // registers per lane: the row rounded up to a multiple of 32 x {8, 32, 64, 96, 128, 192}
  const int vpl = (maxb + 31) / 32;
#define MMDIT_SEL(V) \
  if (vpl <= V) return launch_select_vpl<V>(S, tab_n, B, H, maxb, top_k, top_p, cap, idx, cnt, err, s)
  MMDIT_SEL(8);
  MMDIT_SEL(32);
  MMDIT_SEL(64);
  MMDIT_SEL(96);
  MMDIT_SEL(128);
  MMDIT_SEL(192);
#undef MMDIT_SEL
  return cudaErrorInvalidValue;  // more blocks than the library supports (checked earlier)
}

cudaError_t launch_groups(const int2* tab, const int* tab_n, int B, int maxb, int N, int maxg,
                          int4* groups, int* n_groups, int* err, cudaStream_t s) {
  groups_kernel<<<B, 32, 0, s>>>(tab, tab_n, maxb, N, maxg, groups, n_groups, err);
  return cudaGetLastError();
}

cudaError_t launch_union(const int32_t* idx, const int32_t* cnt, int cap, const int2* tab,
                         const int* tab_n, int maxb, int N, const int4* groups,
                         const int* n_groups, int maxg, int B, int H, int ucap, uint4* ulist,
                         int* ucnt, int* err, cudaStream_t s) {
  if (maxg == 0) return cudaSuccess;
  const size_t smem = sizeof(uint32_t) * (size_t)maxb;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess)
    e = once_per_device(dev, [] {
      return cudaFuncSetAttribute(union_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)(sizeof(uint32_t) * kMaxBlocks));
    });
  if (e != cudaSuccess) return e;
  union_kernel<<<dim3(maxg, H, B), 256, smem, s>>>(idx, cnt, cap, tab, tab_n, maxb, N, groups,
                                                   n_groups, maxg, H, ucap, ulist, ucnt, err);
  return cudaGetLastError();
}

cudaError_t launch_schedule(const int* n_groups, int maxg, int B, int H, int* order,
                            int* n_order, cudaStream_t s) {
  schedule_kernel<<<1, kSchedThreads, 0, s>>>(n_groups, maxg, H, maxg * H * B, order, n_order);
  return cudaGetLastError();
}

}  // namespace mmdit
