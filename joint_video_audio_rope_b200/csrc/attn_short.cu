// Attention of many query rows over a short key sequence (<= 256 keys) on
// the sm_100a tensor cores: the video-query direction of the audio<->video
// cross-attention, video tokens over the 218 audio tokens of the layer
// (SkyReels-V4 digest, arXiv 2602.21818, workflow step 3; SkyReels-V4 blog,
// section 2.2: bidirectional audio-video cross-attention in every block).
//
// O = softmax(Q K^T * scale) V per (batch, head) for bf16 Q/K/V, head_dim
// 128, fp32 accumulation and softmax.  With every key in one tile the softmax
// needs one pass and no running max: per 128-row Q tile,
//   S = Q K^T          one tcgen05.mma group, M = 128, N = 256 (all keys)
//   P = exp(S - max)   one pass over the row (two TMEM reads of S)
//   O = P V            K = the keys rounded up to 16
// Tensor memory per Q tile is 256 columns: S fills them; the softmax writes
// P (bf16, two keys per column) over the first 128 and O accumulates in the
// last 128, which S no longer needs once the softmax has read it.  Two Q
// tiles per CTA (512 columns) ping-pong on the tensor core.  K and V of the
// (batch, head) stay resident in shared memory while the CTA walks the Q
// tiles of that head: each persistent CTA takes a contiguous run of work
// items (pairs of Q tiles) in (batch, head, tile) order and reloads K/V only
// when the head changes.
//
// CTA: warps 0-7 two softmax warpgroups (thread = row = TMEM lane), warp 8
// TMA producer, warp 9 TMEM allocator and MMA issuer, warps 10-11 idle.  No
// TMA multicast.  Every mbarrier wait is bounded (library error word).
#include <math.h>

#include "internal.h"

namespace mmdit {

namespace {

constexpr int kSkThreads = 384;
constexpr int kSkProducerWarp = 8;
constexpr int kSkMmaWarp = 9;
constexpr int kSkMaxKeys = 256;
constexpr int kQTileBytes = 128 * 128 * 2;     // 32 KB: 128 rows x 128 channels
constexpr int kQHalf = 128 * 128;              // one 64-channel half of a Q tile
constexpr int kKVBytes = kSkMaxKeys * 128 * 2; // 64 KB: 256 rows x 128 channels
constexpr int kKVHalf = kSkMaxKeys * 128;      // one 64-channel half of K or V
constexpr int kBox = 64 * 128;                 // one TMA box: 64 rows x 64 channels
constexpr int kStageColsS = 32;                // epilogue: 32 channels per store round
constexpr int kStageWarp = 32 * kStageColsS * 2;
constexpr int kOffK = 0;
constexpr int kOffV = kOffK + kKVBytes;
constexpr int kOffQ = kOffV + kKVBytes;
constexpr int kOffStage = kOffQ + 2 * kQTileBytes;
constexpr int kOffBar = kOffStage + 2 * 8 * kStageWarp;  // two staging buffers per warp
constexpr int kSkSmem = kOffBar + 256 + 1024;
// registers: launched at 168 per thread (384 x 168 = 64,512); the producer /
// MMA warpgroup drops to 104 and the softmax warpgroups rise to 200
constexpr int kSkRegsLow = 104;
constexpr int kSkRegsHigh = 200;
static_assert(128 * (2 * kSkRegsHigh + kSkRegsLow) <= kSkThreads * 168, "register split");

enum {
  SB_QFULL = 0,   // 2
  SB_QEMPTY = 2,  // 2: QK of the tile done (Q buffer reusable)
  SB_KVFULL = 4,  // 1
  SB_KVEMPTY = 5, // 1: every MMA reading the resident K/V done
  SB_SFULL = 6,   // 2
  SB_PFULL = 8,   // 2 (128 arrivals)
  SB_OFULL = 10,  // 2
  SB_OEMPTY = 12, // 2 (128 arrivals): O read out of TMEM
  SB_DONE = 14,   // 1
  SB_COUNT = 15
};

constexpr uint32_t kIdescS = idesc_bf16_f32(128, 256, 0, 0);  // Q, K both K-major
constexpr uint32_t kIdescO = idesc_bf16_f32(128, 128, 0, 1);  // P (TMEM), V MN-major

struct ShortWork {
  int b, h, pair;  // Q rows [256 pair, 256 pair + 256) of head h, batch b
};

// Items (b, h, pair) in order; a CTA's run is [first, last).
__device__ __forceinline__ ShortWork short_item(int item, int pairs, int H) {
  ShortWork w;
  w.pair = item % pairs;
  const int bh = item / pairs;
  w.h = bh % H;
  w.b = bh / H;
  return w;
}

__device__ __forceinline__ void load_rows(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                          int h, int b, int row0, int nbox, int half_bytes) {
  for (int i = 0; i < nbox; ++i) {
    tma_load_4d(dst + i * kBox, map, bar, 0, h, row0 + 64 * i, b);
    tma_load_4d(dst + half_bytes + i * kBox, map, bar, 64, h, row0 + 64 * i, b);
  }
}

__global__ void __launch_bounds__(kSkThreads, 1) attn_short_kernel(const __grid_constant__ AttnParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bars = sbase + kOffBar;
  auto bar = [&](int i) { return bars + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffBar + 8 * SB_COUNT);
  const AttnProblem& pr = P.prob;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* err = P.err;
  const bool skip = *(volatile int*)err != 0;
  const int nkv = pr.Nkv;                       // 1..256
  const int n_chunks = (nkv + 31) >> 5;         // 32-key chunks of S
  const int n_ksteps = (nkv + 15) >> 4;         // K steps of the PV product
  const int pairs = (pr.Nq + 255) >> 8;
  const int items = pairs * pr.H * pr.B;
  const int first = (int)(((long long)items * blockIdx.x) / gridDim.x);
  const int last = (int)(((long long)items * (blockIdx.x + 1)) / gridDim.x);

  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(SB_QFULL + t), 1);
      mbar_init(bar(SB_QEMPTY + t), 1);
      mbar_init(bar(SB_SFULL + t), 1);
      mbar_init(bar(SB_PFULL + t), 128);
      mbar_init(bar(SB_OFULL + t), 1);
      mbar_init(bar(SB_OEMPTY + t), 128);
    }
    mbar_init(bar(SB_KVFULL), 1);
    mbar_init(bar(SB_KVEMPTY), 1);
    mbar_init(bar(SB_DONE), 1);
    fence_mbar_init();
  }
  if (warp == kSkMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 8) {
    setmaxnreg_dec<kSkRegsLow>();
    if (warp == kSkProducerWarp && lane == 0 && !skip) {
      // ---------------------------------------------------------- producer
      tma_prefetch_desc(&pr.tmQ);
      tma_prefetch_desc(&pr.tmK);
      tma_prefetch_desc(&pr.tmV);
      tma_prefetch_desc(&pr.tmO);
      bool ok = true;
      int cur_bh = -1, kv_loads = 0, n = 0;
      const int kv_boxes = (nkv + 63) >> 6;
      for (int it = first; it < last && ok; ++it, ++n) {
        const ShortWork w = short_item(it, pairs, pr.H);
        const int bh = w.b * pr.H + w.h;
        if (bh != cur_bh) {
          if (kv_loads > 0 && !(ok = mbar_wait(bar(SB_KVEMPTY), (kv_loads - 1) & 1, err))) break;
          mbar_expect_tx(bar(SB_KVFULL), 2u * kv_boxes * 2 * kBox);
          load_rows(sbase + kOffK, &pr.tmK, bar(SB_KVFULL), w.h, w.b, 0, kv_boxes, kKVHalf);
          load_rows(sbase + kOffV, &pr.tmV, bar(SB_KVFULL), w.h, w.b, 0, kv_boxes, kKVHalf);
          cur_bh = bh;
          ++kv_loads;
        }
        for (int t = 0; t < 2 && ok; ++t) {
          if (n > 0 && !(ok = mbar_wait(bar(SB_QEMPTY + t), (n - 1) & 1, err))) break;
          mbar_expect_tx(bar(SB_QFULL + t), kQTileBytes);
          load_rows(sbase + kOffQ + t * kQTileBytes, &pr.tmQ, bar(SB_QFULL + t), w.h, w.b,
                    w.pair * 256 + t * 128, 2, kQHalf);
        }
      }
      // every copy issued lands before the CTA's shared memory goes away
      if (n > 0)
        for (int t = 0; t < 2; ++t) mbar_wait(bar(SB_QFULL + t), (n - 1) & 1, err);
      if (kv_loads > 0) mbar_wait(bar(SB_KVFULL), (kv_loads - 1) & 1, err);
    } else if (warp == kSkMmaWarp && lane == 0 && !skip) {
      // ---------------------------------------------------------- MMA issuer
      // Issue order QK_0(n), PV_1(n-1), QK_1(n), PV_0(n), QK_0(n+1), ...: the
      // two tiles run half a period apart, so each softmax overlaps the other
      // tile's PV, epilogue read and QK instead of the other softmax (they
      // would share the MUFU).  QK_t(n) waits for its Q and for the epilogue
      // of item n-1 to have read O_t out (S_t and O_t share TMEM columns).
      bool ok = true;
      int cur_bh = -1, kv_loads = 0;
      const int n_items = last - first;
      auto issue_qk = [&](int t, int n) -> bool {
        if (!mbar_wait(bar(SB_QFULL + t), n & 1, err)) return false;
        if (n > 0 && !mbar_wait(bar(SB_OEMPTY + t), (n - 1) & 1, err)) return false;
        tc_fence_after();
        // eight MMAs of K = 16 channels in one asm block: the descriptors'
        // start-address field (address >> 4) steps by 2 per 32 bytes and by
        // the column-half distance >> 4 at channel 64 (addresses < 256 KB)
        const uint64_t qd = smem_desc_sw128(sbase + kOffQ + t * kQTileBytes, 16, 1024);
        const uint64_t kd = smem_desc_sw128(sbase + kOffK, 16, 1024);
        asm volatile(
            "{\n\t.reg .pred pf, pt;\n\t.reg .b64 ta, tb;\n\t"
            "setp.ne.b32 pf, %3, %3;\n\t"
            "setp.eq.b32 pt, %3, %3;\n\t"
            "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, pf;\n\t"
            "add.s64 ta, %1, 2;\n\tadd.s64 tb, %2, 2;\n\t"
            "tcgen05.mma.cta_group::1.kind::f16 [%0], ta, tb, %3, pt;\n\t"
            "add.s64 ta, %1, 4;\n\tadd.s64 tb, %2, 4;\n\t"
            "tcgen05.mma.cta_group::1.kind::f16 [%0], ta, tb, %3, pt;\n\t"
            "add.s64 ta, %1, 6;\n\tadd.s64 tb, %2, 6;\n\t"
            "tcgen05.mma.cta_group::1.kind::f16 [%0], ta, tb, %3, pt;\n\t"
            "add.s64 ta, %1, %4;\n\tadd.s64 tb, %2, %5;\n\t"
            "tcgen05.mma.cta_group::1.kind::f16 [%0], ta, tb, %3, pt;\n\t"
            "add.s64 ta, ta, 2;\n\tadd.s64 tb, tb, 2;\n\t"
            "tcgen05.mma.cta_group::1.kind::f16 [%0], ta, tb, %3, pt;\n\t"
            "add.s64 ta, ta, 2;\n\tadd.s64 tb, tb, 2;\n\t"
            "tcgen05.mma.cta_group::1.kind::f16 [%0], ta, tb, %3, pt;\n\t"
            "add.s64 ta, ta, 2;\n\tadd.s64 tb, tb, 2;\n\t"
            "tcgen05.mma.cta_group::1.kind::f16 [%0], ta, tb, %3, pt;\n\t}"
            ::"r"(tmem + 256 * t), "l"(qd), "l"(kd), "r"(kIdescS),
            "l"((uint64_t)(kQHalf >> 4)), "l"((uint64_t)(kKVHalf >> 4)));
        tc_commit(bar(SB_SFULL + t));
        tc_commit(bar(SB_QEMPTY + t));
        return true;
      };
      auto issue_pv = [&](int t, int n) -> bool {
        if (!mbar_wait(bar(SB_PFULL + t), n & 1, err)) return false;
        tc_fence_after();
        const uint32_t s_tmem = tmem + 256 * t;
        // 16 key rows (2048 bytes: 128 in the descriptor) and 8 P columns
        // per K step
        const uint64_t vd = smem_desc_sw128(sbase + kOffV, kKVHalf, 1024);
        for (int kk = 0; kk < n_ksteps; ++kk)
          tc_mma_ts(s_tmem + 128, s_tmem + kk * 8, vd + 128u * kk, kIdescO, kk > 0 ? 1u : 0u);
        tc_commit(bar(SB_OFULL + t));
        return true;
      };
      // K/V of item n resident: when the head changes, every MMA issued so far
      // (all of the old head's) completes before the producer reloads K/V
      auto ensure_kv = [&](int n) -> bool {
        const ShortWork w = short_item(first + n, pairs, pr.H);
        const int bh = w.b * pr.H + w.h;
        if (bh == cur_bh) return true;
        if (kv_loads > 0) tc_commit(bar(SB_KVEMPTY));
        if (!mbar_wait(bar(SB_KVFULL), kv_loads & 1, err)) return false;
        cur_bh = bh;
        ++kv_loads;
        return true;
      };
      bool pv1_pending = false;  // PV_1 of the previous item not issued yet
      if (n_items > 0) ok = ensure_kv(0) && issue_qk(0, 0);
      for (int n = 0; n < n_items && ok; ++n) {
        if (pv1_pending) {
          if (!(ok = issue_pv(1, n - 1))) break;
          pv1_pending = false;
        }
        if (!(ok = issue_qk(1, n))) break;
        if (!(ok = issue_pv(0, n))) break;
        pv1_pending = true;
        if (n + 1 < n_items) {
          const ShortWork wn = short_item(first + n + 1, pairs, pr.H);
          if (wn.b * pr.H + wn.h != cur_bh) {  // the old K/V is still read by PV_1(n)
            if (!(ok = issue_pv(1, n))) break;
            pv1_pending = false;
          }
          if (!(ok = ensure_kv(n + 1) && issue_qk(0, n + 1))) break;
        }
      }
      if (ok && pv1_pending) issue_pv(1, n_items - 1);
      tc_commit(bar(SB_DONE));
      mbar_wait(bar(SB_DONE), 0, err);
    }
  } else {
    // ------------------------------------------------------------ softmax
    setmaxnreg_inc<kSkRegsHigh>();
    const int t = warp >> 2;
    const int r = (warp & 3) * 32 + lane;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t s_addr = tmem + lane_off + 256 * t;
    const uint32_t o_addr = s_addr + 128;
    const float sl2 = P.scale_log2;
    const uint64_t sl2x2 = pack_f32x2(sl2, sl2);
    bool ok = !skip;
    int n = 0;
    for (int it = first; it < last && ok; ++it, ++n) {
      const ShortWork w = short_item(it, pairs, pr.H);
      ok = mbar_wait(bar(SB_SFULL + t), n & 1, err);
      if (__any_sync(0xffffffffu, !ok)) {
        ok = false;
        break;
      }
      __syncwarp();
      tc_fence_after();
      // pass 1: the row maximum over the valid keys
      float m = -INFINITY;
      for (int c = 0; c < n_chunks; ++c) {
        uint32_t v[32];
        tmem_ld32(s_addr + 32 * c, v);
        tmem_wait_ld();
        const int valid = nkv - 32 * c;  // keys of this chunk (>= 1)
        float s[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) s[i] = i < valid ? __uint_as_float(v[i]) : -INFINITY;
        float a = max3f(s[0], s[1], s[2]);
#pragma unroll
        for (int i = 3; i + 1 < 32; i += 2) a = max3f(a, s[i], s[i + 1]);
        m = fmaxf(m, fmaxf(a, s[31]));
      }
      // pass 2: probabilities (bf16, over the first columns of S) and their sum
      const float mref = m * sl2;
      const uint64_t nm2 = pack_f32x2(-mref, -mref);
      uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
      for (int c = 0; c < n_chunks; ++c) {
        uint32_t v[32];
        tmem_ld32(s_addr + 32 * c, v);
        tmem_wait_ld();
        const int valid = nkv - 32 * c;
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint64_t x2 = ffma_f32x2(pack_f32x2(__uint_as_float(v[2 * i]),
                                                    __uint_as_float(v[2 * i + 1])), sl2x2, nm2);
          float p0, p1;
          unpack_f32x2(x2, p0, p1);
          p0 = 2 * i < valid ? ex2_approx(p0) : 0.f;
          p1 = 2 * i + 1 < valid ? ex2_approx(p1) : 0.f;
          pk[i] = pack_bf16x2(p0, p1);
          acc[i & 3] = add_f32x2(acc[i & 3], pack_f32x2(p0, p1));
        }
        tmem_st16(s_addr + 16 * c, pk);
      }
      // keys past the last chunk up to the PV product's K (a multiple of 16)
      // are already zero: n_ksteps * 16 <= n_chunks * 32
      tmem_wait_st();
      float l;
      {
        float a0, a1, b0, b1;
        unpack_f32x2(add_f32x2(acc[0], acc[1]), a0, a1);
        unpack_f32x2(add_f32x2(acc[2], acc[3]), b0, b1);
        l = (a0 + a1) + (b0 + b1);
      }
      tc_fence_before();
      mbar_arrive(bar(SB_PFULL + t));

      // ---------------------------------------------------------- epilogue
      ok = mbar_wait(bar(SB_OFULL + t), n & 1, err);
      if (__any_sync(0xffffffffu, !ok)) {
        ok = false;
        break;
      }
      __syncwarp();
      tc_fence_after();
      uint32_t o0[32], o1[32], o2[32], o3[32];
      tmem_ld32(o_addr, o0);
      tmem_ld32(o_addr + 32, o1);
      tmem_ld32(o_addr + 64, o2);
      tmem_ld32(o_addr + 96, o3);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bar(SB_OEMPTY + t));
      const float inv = l > 0.f ? 1.f / l : 0.f;
      auto ov = [&](int c) -> uint32_t {
        return c < 32 ? o0[c] : c < 64 ? o1[c - 32] : c < 96 ? o2[c - 64] : o3[c - 96];
      };
      const int row0 = w.pair * 256 + t * 128;  // first query row of this tile
      const int qrow = row0 + r;
      if (pr.row_sq != nullptr && qrow < pr.Nq) {
        float ss = 0.f;
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          const float x = __uint_as_float(ov(c)) * inv;
          ss = fmaf(x, x, ss);
        }
        pr.row_sq[((long long)w.b * pr.Nq + qrow) * pr.H + w.h] = ss;
      }
      const int wrow = row0 + (warp & 3) * 32;  // first row of this warp
      if (wrow < pr.Nq) {
        const int sw = ((lane * kStageColsS * 2) >> 7) & 3;  // 64-byte swizzle of this lane's row
#pragma unroll
        for (int rr = 0; rr < 128 / kStageColsS; ++rr) {
          // two staging buffers per warp: a round waits only for the store
          // issued two rounds ago to have read its buffer
          uint8_t* stg = smem + kOffStage + (2 * warp + (rr & 1)) * kStageWarp;
          if (lane == 0) bulk_wait_read<1>();
          __syncwarp();
#pragma unroll
          for (int chunk = 0; chunk < 4; ++chunk) {
            const int c0 = rr * kStageColsS + chunk * 8;
            uint4 q4;
            q4.x = pack_bf16x2(__uint_as_float(ov(c0 + 0)) * inv, __uint_as_float(ov(c0 + 1)) * inv);
            q4.y = pack_bf16x2(__uint_as_float(ov(c0 + 2)) * inv, __uint_as_float(ov(c0 + 3)) * inv);
            q4.z = pack_bf16x2(__uint_as_float(ov(c0 + 4)) * inv, __uint_as_float(ov(c0 + 5)) * inv);
            q4.w = pack_bf16x2(__uint_as_float(ov(c0 + 6)) * inv, __uint_as_float(ov(c0 + 7)) * inv);
            *reinterpret_cast<uint4*>(stg + lane * (kStageColsS * 2) + ((chunk ^ sw) << 4)) = q4;
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_4d(&pr.tmO, smem_u32(stg), rr * kStageColsS, w.h, wrow, w.b);
            bulk_commit();
          }
        }
      }
    }
  }

  // ------------------------------------------------------------ teardown
  bulk_wait<0>();
  tc_fence_before();
  __syncthreads();
  if (warp == kSkMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

int attn_short_store_cols() { return kStageColsS; }

cudaError_t launch_attn_short(const AttnParams& p, cudaStream_t s) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = once_per_device(dev, [] {
    return cudaFuncSetAttribute(attn_short_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                kSkSmem);
  });
  if (e != cudaSuccess) return e;
  const AttnProblem& pr = p.prob;
  if (pr.Nkv < 1 || pr.Nkv > kSkMaxKeys) return cudaErrorInvalidValue;
  const long long items = (long long)((pr.Nq + 255) / 256) * pr.H * pr.B;
  if (items == 0) return cudaSuccess;
  int sms = 0;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int grid = (int)std::min<long long>(items, sms);
  attn_short_kernel<<<grid, kSkThreads, kSkSmem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace mmdit
