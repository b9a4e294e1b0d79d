// Content-adaptive block shapes of the block-sparse mode (Prism guide, arXiv
// 2610.05416, Key ideas and Method sections 1-2).
//
// The T x H x W token volume of a raster-order video is cut into macro-zones
// of 8 x 8 x 8 tokens (zones on the far edge of an axis are short).  Per zone
// m, from the value features V (all heads and channels, D = heads x 128):
//   sigma^2_{v,d}(m) = (1/D) sum_c (1/Z_d) sum_i (Vbar^(d)_{m,i,c} - mu^(d)_{m,c})^2
// with Vbar^(d)_{m,i} the mean of V over the zone's tokens with index i along
// axis d and mu^(d) the mean of those slice means; r_{v,d} = sigma^2_{v,d} /
// sum_d' sigma^2_{v,d'}.  From the A->V cross-attention output norms a of the
// preceding layer: abar(m) (the zone mean of a over the largest zone mean)
// and vhat_{a,d}(m) (the directional variance of a, normalised like r).
//   g_d(m) = r_{v,d}(m) + abar(m) vhat_{a,d}(m) + eps
// The zone's density rho(m) = sum_d sigma^2_{v,d}(m) / (its maximum over the
// zones) picks the block volume B(m) = 64 (rho >= tau_128), 128 (rho >=
// tau_256) or 256, and the block shape is the candidate of that volume (edges
// 2, 4 or 8 with product B: 7 + 6 + 3 = 16 shapes) nearest in log2 space to
//   l*_d = -1/2 log2 g_d + 1/3 (log2 B + 1/2 sum_d' log2 g_d').
// The zone is cut into blocks of that shape (clipped at its edge).  Storage
// order: zones in raster order, a zone's blocks in raster order, a block's
// tokens in (t, h, w) raster order, so every block is one contiguous run.
//
// Kernels:
//   zone_stats_kernel  one CTA per (zone, head, batch), one warp per t-slice:
//                      slice sums of the head's 128 channels along t, h and w
//                      (fp32, lane = 4 channels) and the three centred
//                      variance sums; the head-0 CTA also takes the
//                      statistics of the norms a.
//   zone_plan_kernel   one CTA per batch item: the indicator, volume and shape
//                      of every zone in fp64, the zone and block prefix sums,
//                      the block table and the zone table.
//   permute_kernel     one warp per token row: raster <-> adaptive storage
//                      order of up to three [B, N, heads, 128] tensors.
//   cross_norm_kernel  a_{t,h,w} = sqrt of the sum over heads of the squared
//                      per-head norms the cross-attention epilogue wrote.
#include <math.h>

#include "internal.h"

namespace mmdit {

namespace {

constexpr int kZone = 8;
constexpr int kPlanThreads = 1024;

// the 16 candidate shapes (b_T, b_H, b_W): volume 64 (7), 128 (6), 256 (3),
// each volume's shapes in ascending lexicographic order (distance ties go to
// the earlier one)
__constant__ int8_t c_shapes[16][3] = {
    {2, 4, 8}, {2, 8, 4}, {4, 2, 8}, {4, 4, 4}, {4, 8, 2}, {8, 2, 4}, {8, 4, 2},
    {2, 8, 8}, {4, 4, 8}, {4, 8, 4}, {8, 2, 8}, {8, 4, 4}, {8, 8, 2},
    {4, 8, 8}, {8, 4, 8}, {8, 8, 4}};

struct ZoneGrid {
  int T, H, W, nzt, nzh, nzw;
  __host__ __device__ int count() const { return nzt * nzh * nzw; }
  __device__ void zone(int z, int& t0, int& h0, int& w0, int& et, int& eh, int& ew) const {
    const int zt = z / (nzh * nzw), r = z - zt * nzh * nzw, zh = r / nzw, zw = r - zh * nzw;
    t0 = zt * kZone;
    h0 = zh * kZone;
    w0 = zw * kZone;
    et = min(kZone, T - t0);
    eh = min(kZone, H - h0);
    ew = min(kZone, W - w0);
  }
};

ZoneGrid zone_grid(int T, int H, int W) {
  return ZoneGrid{T, H, W, (T + kZone - 1) / kZone, (H + kZone - 1) / kZone, (W + kZone - 1) / kZone};
}

__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Centred variance sum of `n` slice means m_i = s_i / cnt:  sum_i (m_i - mu)^2.
template <int NMAX>
__device__ __forceinline__ float centred(const float (&s)[NMAX], int n, float cnt) {
  float mu = 0.f;
#pragma unroll
  for (int i = 0; i < NMAX; ++i) mu += i < n ? s[i] / cnt : 0.f;
  mu /= (float)n;
  float v = 0.f;
#pragma unroll
  for (int i = 0; i < NMAX; ++i) {
    const float d = s[i] / cnt - mu;
    v += i < n ? d * d : 0.f;
  }
  return v;
}

// Centred variance sum of `n` means m_i:  sum_i (m_i - mu)^2, mu = mean of m_i.
template <int NMAX>
__device__ __forceinline__ float centred_means(const float (&m)[NMAX], int n) {
  float mu = 0.f;
#pragma unroll
  for (int i = 0; i < NMAX; ++i) mu += i < n ? m[i] : 0.f;
  mu /= (float)n;
  float v = 0.f;
#pragma unroll
  for (int i = 0; i < NMAX; ++i) {
    const float d = m[i] - mu;
    v += i < n ? d * d : 0.f;
  }
  return v;
}

// part[b][z][h][3] = sum over the head's channels of (1/Z_d) sum_i (slice mean
// - mean)^2 along t, h, w;  ast[b][z][4] = the same three for the norms a (a
// single channel) and the zone mean of a (zeros when a is NULL).
// One CTA per (zone, head, batch), one warp per t-slice of the zone (lane =
// 4 channels): each warp sums its slice, its slice's rows (h) and columns
// (w); warp 0 combines the warps' partial h and w sums from shared memory.
constexpr int kStatsThreads = 32 * kZone;
constexpr int kStatsSmem = (int)sizeof(float) * (kZone * 128 + 2 * kZone * kZone * 128);

__global__ void __launch_bounds__(kStatsThreads, 2) zone_stats_kernel(
    const __nv_bfloat16* __restrict__ v, long long st, long long sb, int heads, ZoneGrid zg,
    const float* __restrict__ a, float* __restrict__ part, float* __restrict__ ast) {
  extern __shared__ float s_dyn[];
  float(*s_t)[128] = reinterpret_cast<float(*)[128]>(s_dyn);                  // [t] slice sums
  float(*s_h)[kZone][128] = reinterpret_cast<float(*)[kZone][128]>(s_dyn + kZone * 128);  // [warp][h]
  float(*s_w)[kZone][128] =
      reinterpret_cast<float(*)[kZone][128]>(s_dyn + kZone * 128 + kZone * kZone * 128);  // [warp][w]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // heads are the fastest grid dimension: the CTAs of one zone run side by
  // side and read whole token rows (every head's 256 bytes) together
  const int h = blockIdx.x, z = blockIdx.y, b = blockIdx.z;
  const int nz = zg.count();
  int t0, h0, w0, et, eh, ew;
  zg.zone(z, t0, h0, w0, et, eh, ew);
  const int lt = warp;  // this warp's t-slice
  float sh[kZone][4], sw[kZone][4], stt[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int i = 0; i < kZone; ++i)
#pragma unroll
    for (int c = 0; c < 4; ++c) sh[i][c] = sw[i][c] = 0.f;
  if (lt < et) {
    const __nv_bfloat16* base = v + (long long)b * sb + (long long)h * 128 + 4 * lane;
    // the slice's 8 x 8 tokens in two halves of four rows (32 loads in flight)
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      uint2 raw[kZone / 2][kZone];
#pragma unroll
      for (int i = 0; i < kZone / 2; ++i) {
        const int lh = half * (kZone / 2) + i;
        const long long row = ((long long)(t0 + lt) * zg.H + (h0 + lh)) * zg.W + w0;
#pragma unroll
        for (int lw = 0; lw < kZone; ++lw)
          raw[i][lw] = (lh < eh && lw < ew)
                           ? __ldg(reinterpret_cast<const uint2*>(base + (row + lw) * st))
                           : make_uint2(0u, 0u);
      }
#pragma unroll
      for (int i = 0; i < kZone / 2; ++i) {
        const int lh = half * (kZone / 2) + i;
#pragma unroll
        for (int lw = 0; lw < kZone; ++lw) {
          const float2 x01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw[i][lw].x));
          const float2 x23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw[i][lw].y));
          const float x[4] = {x01.x, x01.y, x23.x, x23.y};
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            sh[lh][c] += x[c];
            sw[lw][c] += x[c];
            stt[c] += x[c];
          }
        }
      }
    }
  }
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    s_t[lt][4 * lane + c] = stt[c];
#pragma unroll
    for (int i = 0; i < kZone; ++i) {
      s_h[lt][i][4 * lane + c] = sh[i][c];
      s_w[lt][i][4 * lane + c] = sw[i][c];
    }
  }
  __syncthreads();
  // the centred variance sums, one channel per thread: threads 0-127 take the
  // t and h axes of channel tid, threads 128-255 the w axis of channel tid-128
  // (slice means as sums times the reciprocal of the slice's token count)
  {
    const int c = threadIdx.x & 127, part_id = threadIdx.x >> 7;
    float m8[kZone], va = 0.f, vb = 0.f;
    if (part_id == 0) {
      const float it = 1.f / (float)(eh * ew), ih = 1.f / (float)(et * ew);
#pragma unroll
      for (int i = 0; i < kZone; ++i) m8[i] = s_t[i][c] * it;
      va = centred_means(m8, et) / (float)et;
#pragma unroll
      for (int i = 0; i < kZone; ++i) {
        float hs = 0.f;
#pragma unroll
        for (int k = 0; k < kZone; ++k) hs += s_h[k][i][c];  // over the t-slices, in order
        m8[i] = hs * ih;
      }
      vb = centred_means(m8, eh) / (float)eh;
    } else {
      const float iw = 1.f / (float)(et * eh);
#pragma unroll
      for (int i = 0; i < kZone; ++i) {
        float ws = 0.f;
#pragma unroll
        for (int k = 0; k < kZone; ++k) ws += s_w[k][i][c];
        m8[i] = ws * iw;
      }
      va = centred_means(m8, ew) / (float)ew;
    }
    // sums over the head's 128 channels: warps, then the four warps of a part
    va = warp_sum_f(va);
    vb = warp_sum_f(vb);
    __shared__ float s_red[kZone][2];
    if (lane == 0) {
      s_red[warp][0] = va;
      s_red[warp][1] = vb;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      float vt = 0.f, vh = 0.f, vw = 0.f;
      for (int w_ = 0; w_ < 4; ++w_) {
        vt += s_red[w_][0];
        vh += s_red[w_][1];
        vw += s_red[4 + w_][0];
      }
      float* o = part + (((long long)b * nz + z) * heads + h) * 3;
      o[0] = vt;
      o[1] = vh;
      o[2] = vw;
    }
  }
  if (h != 0 || warp != 1) return;
  // statistics of the norms a of this zone (warp 1 of the head-0 CTA): lane l
  // takes the tokens l, l+32, ...
  float at[kZone], ah[kZone], aw[kZone], asum = 0.f;
#pragma unroll
  for (int i = 0; i < kZone; ++i) at[i] = ah[i] = aw[i] = 0.f;
  if (a != nullptr) {
    const int n = et * eh * ew;
    for (int i = lane; i < n; i += 32) {
      const int lt2 = i / (eh * ew), r = i - lt2 * eh * ew, lh = r / ew, lw = r - lh * ew;
      const float x = a[(long long)b * zg.T * zg.H * zg.W +
                        ((long long)(t0 + lt2) * zg.H + (h0 + lh)) * zg.W + (w0 + lw)];
#pragma unroll
      for (int k = 0; k < kZone; ++k) {
        at[k] += k == lt2 ? x : 0.f;
        ah[k] += k == lh ? x : 0.f;
        aw[k] += k == lw ? x : 0.f;
      }
      asum += x;
    }
#pragma unroll
    for (int k = 0; k < kZone; ++k) {
      at[k] = warp_sum_f(at[k]);
      ah[k] = warp_sum_f(ah[k]);
      aw[k] = warp_sum_f(aw[k]);
    }
    asum = warp_sum_f(asum);
  }
  if (lane == 0) {
    float* o = ast + ((long long)b * nz + z) * 4;
    o[0] = centred(at, et, (float)(eh * ew)) / (float)et;
    o[1] = centred(ah, eh, (float)(et * ew)) / (float)eh;
    o[2] = centred(aw, ew, (float)(et * eh)) / (float)ew;
    o[3] = asum / (float)(et * eh * ew);
  }
}

// Block-wide exclusive scan of one int per thread (kPlanThreads threads);
// returns the exclusive prefix and the total.
__device__ int plan_scan(int v, int* ws, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += t;
  }
  if (lane == 31) ws[warp] = x;
  __syncthreads();
  int before = 0;
  total = 0;
  for (int w = 0; w < kPlanThreads / 32; ++w) {
    before += w < warp ? ws[w] : 0;
    total += ws[w];
  }
  __syncthreads();
  return before + x - v;
}

// One CTA per batch item.  zones[b][z] = {shape 0..15, first storage token,
// first block, blocks}; blocks[b][i] = {start, length}; n_blocks[b].
__global__ void __launch_bounds__(kPlanThreads) zone_plan_kernel(
    const float* __restrict__ part, const float* __restrict__ ast, int heads, ZoneGrid zg,
    float tau128, float tau256, float eps, int has_a, int max_blocks, int4* __restrict__ zones,
    int2* __restrict__ blocks, int* __restrict__ n_blocks, int* err) {
  __shared__ float s_max[2][kPlanThreads / 32];
  __shared__ int s_scan[kPlanThreads / 32];
  const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nz = zg.count();
  const double D = (double)heads * 128.0;
  // pass 1: the largest total variance and the largest zone mean of a
  float tmax = 0.f, amax = 0.f;
  for (int z = tid; z < nz; z += kPlanThreads) {
    const float* p = part + ((long long)b * nz + z) * heads * 3;
    double tot = 0.0;
    for (int h = 0; h < heads; ++h) tot += (double)p[3 * h] + p[3 * h + 1] + p[3 * h + 2];
    tmax = fmaxf(tmax, (float)(tot / D));
    amax = fmaxf(amax, ast[((long long)b * nz + z) * 4 + 3]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, o));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  }
  if (lane == 0) {
    s_max[0][warp] = tmax;
    s_max[1][warp] = amax;
  }
  __syncthreads();
  tmax = amax = 0.f;
  for (int w = 0; w < kPlanThreads / 32; ++w) {
    tmax = fmaxf(tmax, s_max[0][w]);
    amax = fmaxf(amax, s_max[1][w]);
  }
  __syncthreads();
  // pass 2: every zone's plan, in chunks of kPlanThreads zones with running
  // token and block offsets
  int tok_run = 0, blk_run = 0;
  for (int z0 = 0; z0 < nz; z0 += kPlanThreads) {
    const int z = z0 + tid;
    int shape = 0, nblk = 0, ntok = 0, et = 0, eh = 0, ew = 0, t0, h0, w0;
    if (z < nz) {
      zg.zone(z, t0, h0, w0, et, eh, ew);
      const float* p = part + ((long long)b * nz + z) * heads * 3;
      double sig[3] = {0.0, 0.0, 0.0};
      for (int h = 0; h < heads; ++h)
        for (int d = 0; d < 3; ++d) sig[d] += (double)p[3 * h + d];
      for (int d = 0; d < 3; ++d) sig[d] /= D;
      const double tot = sig[0] + sig[1] + sig[2];
      const float* q = ast + ((long long)b * nz + z) * 4;
      const double atot = has_a ? (double)q[0] + q[1] + q[2] : 0.0;
      const double abar = (has_a && amax > 0.f) ? (double)q[3] / (double)amax : 0.0;
      const double rho = tmax > 0.f ? tot / (double)tmax : 0.0;
      double g[3], lsum = 0.0;
      for (int d = 0; d < 3; ++d) {
        const double r = tot > 0.0 ? sig[d] / tot : 0.0;
        const double va = atot > 0.0 ? (double)q[d] / atot : 0.0;
        g[d] = r + abar * va + (double)eps;
        lsum += log2(g[d]);
      }
      const int vol = rho >= (double)tau128 ? 64 : (rho >= (double)tau256 ? 128 : 256);
      const int first = vol == 64 ? 0 : (vol == 128 ? 7 : 13);
      const int count = vol == 64 ? 7 : (vol == 128 ? 6 : 3);
      const double S = vol == 64 ? 6.0 : (vol == 128 ? 7.0 : 8.0);
      double best = 0.0;
      for (int c = first; c < first + count; ++c) {
        double dist = 0.0;
        for (int d = 0; d < 3; ++d) {
          const double l = -0.5 * log2(g[d]) + (S + 0.5 * lsum) / 3.0;
          const double e = log2((double)c_shapes[c][d]) - l;
          dist += e * e;
        }
        if (c == first || dist < best) {
          best = dist;
          shape = c;
        }
      }
      nblk = ((et + c_shapes[shape][0] - 1) / c_shapes[shape][0]) *
             ((eh + c_shapes[shape][1] - 1) / c_shapes[shape][1]) *
             ((ew + c_shapes[shape][2] - 1) / c_shapes[shape][2]);
      ntok = et * eh * ew;
    }
    int tok_total, blk_total;
    const int tok0 = tok_run + plan_scan(ntok, s_scan, tok_total);
    const int blk0 = blk_run + plan_scan(nblk, s_scan, blk_total);
    if (z < nz) {
      zones[(long long)b * nz + z] = make_int4(shape, tok0, blk0, nblk);
      // the zone's blocks in (bt, bh, bw) raster order
      const int bT = c_shapes[shape][0], bH = c_shapes[shape][1], bW = c_shapes[shape][2];
      int i = blk0, start = tok0;
      for (int lt = 0; lt < et; lt += bT)
        for (int lh = 0; lh < eh; lh += bH)
          for (int lw = 0; lw < ew; lw += bW) {
            const int len = min(bT, et - lt) * min(bH, eh - lh) * min(bW, ew - lw);
            MMDIT_DCHECK(i < max_blocks, err);
            if (i < max_blocks) blocks[(long long)b * max_blocks + i] = make_int2(start, len);
            ++i;
            start += len;
          }
    }
    tok_run += tok_total;
    blk_run += blk_total;
  }
  if (tid == 0) n_blocks[b] = min(blk_run, max_blocks);
}

// Storage position of raster token (t, h, w) in the adaptive order.
__device__ __forceinline__ int storage_index(const ZoneGrid& zg, const int4* zones, int t, int h,
                                             int w) {
  const int zt = t / kZone, zh = h / kZone, zw = w / kZone;
  const int z = (zt * zg.nzh + zh) * zg.nzw + zw;
  const int4 zi = zones[z];
  const int et = min(kZone, zg.T - zt * kZone), eh = min(kZone, zg.H - zh * kZone),
            ew = min(kZone, zg.W - zw * kZone);
  const int shape = min(max(zi.x, 0), 15);
  const int bT = c_shapes[shape][0], bH = c_shapes[shape][1], bW = c_shapes[shape][2];
  const int lt = t - zt * kZone, lh = h - zh * kZone, lw = w - zw * kZone;
  const int i = lt / bT, j = lh / bH, k = lw / bW;
  const int xt = min(bT, et - i * bT), xh = min(bH, eh - j * bH), xw = min(bW, ew - k * bW);
  return zi.y + i * bT * eh * ew + xt * j * bH * ew + xt * xh * k * bW +
         ((lt - i * bT) * xh + (lh - j * bH)) * xw + (lw - k * bW);
}

struct PermuteArgs {
  const uint4* src[3];
  uint4* dst[3];
  int n;  // tensors (1..3)
};

// One warp per raster token row: inverse = 0 moves the row to its storage
// position (dst[s] = src[r]), inverse = 1 back (dst[r] = src[s]).  Rows of
// heads * 128 bf16 in 16-byte vectors; strides in 16-byte units.
__global__ void __launch_bounds__(256) permute_kernel(PermuteArgs pa, long long st, long long sb,
                                                      int row_u4, ZoneGrid zg,
                                                      const int4* __restrict__ zones, int inverse,
                                                      int* err) {
  const int b = blockIdx.y;
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int N = zg.T * zg.H * zg.W;
  if (r >= N) return;
  const int lane = threadIdx.x & 31;
  const int t = r / (zg.H * zg.W), rem = r - t * zg.H * zg.W, h = rem / zg.W, w = rem - h * zg.W;
  const int s = storage_index(zg, zones + (long long)b * zg.count(), t, h, w);
  // a zone table that is not a plan of this grid must not move rows outside it
  MMDIT_DCHECK(s >= 0 && s < N, err);
  if (s < 0 || s >= N) return;
  const long long from = b * sb + (long long)(inverse ? s : r) * st;
  const long long to = b * sb + (long long)(inverse ? r : s) * st;
  for (int x = 0; x < pa.n; ++x)
    for (int c = lane; c < row_u4; c += 32) pa.dst[x][to + c] = pa.src[x][from + c];
}

}  // namespace

// a[b][n] = sqrt(sum over heads of sq[b][n][h]) (fixed summation order)
__global__ void cross_norm_kernel(const float* __restrict__ sq, int heads, long long n_rows,
                                  float* __restrict__ a) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_rows) return;
  float s = 0.f;
  for (int h = 0; h < heads; ++h) s += sq[i * heads + h];
  a[i] = sqrtf(s);
}

cudaError_t launch_cross_norms(const float* sq, int heads, long long n_rows, float* a,
                               cudaStream_t s) {
  if (n_rows == 0) return cudaSuccess;
  cross_norm_kernel<<<(unsigned)((n_rows + 255) / 256), 256, 0, s>>>(sq, heads, n_rows, a);
  return cudaGetLastError();
}

namespace {

struct PlanWs {
  size_t part, ast, bytes;
};
PlanWs plan_ws(int B, int heads, int nz) {
  PlanWs w{};
  w.part = 0;
  w.ast = align256(sizeof(float) * (size_t)B * nz * heads * 3);
  w.bytes = w.ast + align256(sizeof(float) * (size_t)B * nz * 4);
  return w;
}

int check_grid(const mmdit_tensor_desc* desc, int T, int H, int W, const char* name) {
  int rc = check_desc(desc, name);
  if (rc) return rc;
  if (desc->dtype != MMDIT_BF16) return fail(MMDIT_EUNSUPPORTED, "%s: bf16 only", name);
  if (T < 1 || H < 1 || W < 1 || (long long)T * H * W != desc->n_tokens)
    return fail(MMDIT_EINVAL, "%s: T*H*W must equal n_tokens", name);
  if (desc->batch > 65535) return fail(MMDIT_EINVAL, "%s: batch %d > 65535", name, desc->batch);
  return MMDIT_OK;
}

}  // namespace

}  // namespace mmdit

using namespace mmdit;

extern "C" {

int mmdit_adaptive_num_zones(int T, int H, int W) {
  if (T < 1 || H < 1 || W < 1) return 0;
  const long long n = (long long)((T + 7) / 8) * ((H + 7) / 8) * ((W + 7) / 8);
  return n > 0x7fffffffLL ? 0 : (int)n;
}

int mmdit_adaptive_max_blocks(int T, int H, int W) {
  const long long nz = mmdit_adaptive_num_zones(T, H, W);
  return 8 * nz > 0x7fffffffLL ? 0 : (int)(8 * nz);
}

size_t mmdit_adaptive_plan_workspace_size(const mmdit_tensor_desc* desc, int T, int H, int W) {
  if (check_grid(desc, T, H, W, "adaptive_plan")) return 0;
  return plan_ws(desc->batch, desc->heads, mmdit_adaptive_num_zones(T, H, W)).bytes;
}

int mmdit_adaptive_plan(const void* v, const float* a_norm, const mmdit_tensor_desc* desc, int T,
                        int H, int W, const mmdit_adaptive_params* params, int32_t* zones,
                        int32_t* blocks, int32_t* n_blocks, int max_blocks, void* workspace,
                        size_t ws_bytes, mmdit_stream_t stream) {
  MMDIT_NVTX("mmdit_adaptive_plan");
  int rc = check_grid(desc, T, H, W, "adaptive_plan");
  if (rc) return rc;
  if (!v || !zones || !blocks || !n_blocks)
    return fail(MMDIT_EINVAL, "adaptive_plan: v, zones, blocks, n_blocks must be non-NULL");
  if (!aligned16(v) || (reinterpret_cast<uintptr_t>(zones) & 15u) ||
      (reinterpret_cast<uintptr_t>(blocks) & 7u) || (a_norm && (reinterpret_cast<uintptr_t>(a_norm) & 3u)))
    return fail(MMDIT_EINVAL, "adaptive_plan: misaligned pointer");
  const int nz = mmdit_adaptive_num_zones(T, H, W);
  if (max_blocks < 8 * nz)
    return fail(MMDIT_EINVAL, "adaptive_plan: max_blocks %d < 8 x %d zones", max_blocks, nz);
  if (8 * nz > kMaxBlocks)
    return fail(MMDIT_EUNSUPPORTED, "adaptive_plan: %d zones may need more than %d blocks", nz,
                kMaxBlocks);
  mmdit_adaptive_params pr{0.5f, 0.25f, 1e-6f};
  if (params != nullptr) pr = *params;
  if (!(pr.tau_256 >= 0.f && pr.tau_256 <= pr.tau_128 && pr.tau_128 <= 1.f) || !(pr.eps > 0.f) ||
      !isfinite(pr.eps))
    return fail(MMDIT_EINVAL, "adaptive_plan: need 0 <= tau_256 <= tau_128 <= 1 and eps > 0");
  const PlanWs w = plan_ws(desc->batch, desc->heads, nz);
  if (workspace == nullptr || ws_bytes < w.bytes)
    return fail(MMDIT_EWORKSPACE, "adaptive_plan: workspace needs %zu bytes", w.bytes);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(MMDIT_EINVAL, "adaptive_plan: workspace must be 256-byte aligned");
  if ((rc = check_sm100())) return rc;
  int* err = device_error_flag();
  if (err == nullptr) return fail(MMDIT_ECUDA, "device error flag unavailable");
  char* ws = static_cast<char*>(workspace);
  float* part = reinterpret_cast<float*>(ws + w.part);
  float* ast = reinterpret_cast<float*>(ws + w.ast);
  const ZoneGrid zg = zone_grid(T, H, W);
  cudaStream_t s = (cudaStream_t)stream;
  int dev = 0;
  cudaError_t e0 = cudaGetDevice(&dev);
  if (e0 == cudaSuccess)
    e0 = once_per_device(dev, [] {
      return cudaFuncSetAttribute(zone_stats_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  kStatsSmem);
    });
  if (e0 != cudaSuccess) return cuda_fail(e0, "adaptive_plan attribute");
  zone_stats_kernel<<<dim3(desc->heads, nz, desc->batch), kStatsThreads, kStatsSmem, s>>>(
      (const __nv_bfloat16*)v, desc->stride_tok, desc->stride_batch, desc->heads, zg, a_norm,
      part, ast);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) {
    zone_plan_kernel<<<desc->batch, kPlanThreads, 0, s>>>(
        part, ast, desc->heads, zg, pr.tau_128, pr.tau_256, pr.eps, a_norm != nullptr,
        max_blocks, reinterpret_cast<int4*>(zones), reinterpret_cast<int2*>(blocks), n_blocks, err);
    e = cudaGetLastError();
  }
  return e == cudaSuccess ? MMDIT_OK : cuda_fail(e, "adaptive_plan launch");
}

int mmdit_adaptive_permute(const void* const* src, void* const* dst, int n_tensors,
                           const mmdit_tensor_desc* desc, int T, int H, int W,
                           const int32_t* zones, int inverse, mmdit_stream_t stream) {
  MMDIT_NVTX("mmdit_adaptive_permute");
  int rc = check_grid(desc, T, H, W, "adaptive_permute");
  if (rc) return rc;
  if (n_tensors < 1 || n_tensors > 3 || src == nullptr || dst == nullptr || zones == nullptr)
    return fail(MMDIT_EINVAL, "adaptive_permute: 1..3 tensors, zones non-NULL");
  if ((reinterpret_cast<uintptr_t>(zones) & 15u) != 0)
    return fail(MMDIT_EINVAL, "adaptive_permute: zones must be 16-byte aligned");
  PermuteArgs pa{};
  pa.n = n_tensors;
  for (int i = 0; i < n_tensors; ++i) {
    if (src[i] == nullptr || dst[i] == nullptr || !aligned16(src[i]) || !aligned16(dst[i]))
      return fail(MMDIT_EINVAL, "adaptive_permute: tensors must be non-NULL and 16-byte aligned");
    if (src[i] == dst[i]) return fail(MMDIT_EINVAL, "adaptive_permute: dst aliases src");
    pa.src[i] = static_cast<const uint4*>(src[i]);
    pa.dst[i] = static_cast<uint4*>(dst[i]);
  }
  if (desc->n_tokens == 0) return MMDIT_OK;
  if ((rc = check_sm100())) return rc;
  int* err = device_error_flag();
  if (err == nullptr) return fail(MMDIT_ECUDA, "device error flag unavailable");
  const ZoneGrid zg = zone_grid(T, H, W);
  permute_kernel<<<dim3((desc->n_tokens + 7) / 8, desc->batch), 256, 0, (cudaStream_t)stream>>>(
      pa, desc->stride_tok / 8, desc->stride_batch / 8, desc->heads * 16, zg,
      reinterpret_cast<const int4*>(zones), inverse != 0, err);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MMDIT_OK : cuda_fail(e, "adaptive_permute launch");
}

}  // extern "C"
