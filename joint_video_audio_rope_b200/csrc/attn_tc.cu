// Flash-style attention on the sm_100a tensor cores (tcgen05 + tensor memory).
//
// Computes O = softmax(Q K^T * scale) V for bf16 Q/K/V with head_dim 128 and
// fp32 accumulation and softmax state.  One kernel serves every attention of
// the layer:
//   * joint self-attention over the concatenated sequence (SkyReels-V4 digest,
//     arXiv 2602.21818, workflow step 3; SkyReels-V4 blog, section 2.1);
//   * the audio-query direction of the audio<->video cross-attention (same
//     sources; blog section 2.2), the video keys split across CTAs and merged
//     afterwards (split-KV); the video-query direction, over at most 256
//     audio keys, has its own kernel (attn_short.cu);
//   * the reinforced text cross-attention (video queries over the text keys,
//     one-tile CTAs, two per SM);
//   * block-sparse attention restricted to selected key blocks (Prism guide,
//     arXiv 2610.05416, Method section 3: online-softmax attention over S_i).
//
// CTA organisation (384 threads = 3 warpgroups, one CTA per SM, for two Q
// tiles; the one-tile shape has 256 threads and two CTAs per SM):
//   warps 0-3  softmax warpgroup for Q tile 0 (128 query rows; thread = row)
//   warps 4-7  softmax warpgroup for Q tile 1
//   warp 8     TMA producer: Q tiles once, then K/V tiles into a 4-slot ring
//   warp 9     tensor-memory allocator and single-thread tcgen05.mma issuer
//   warps 10-11 no role (setmaxnreg hands registers out per warpgroup)
// Tensor memory (512 columns x 128 lanes of 32 bit):
//   [0,128) S0 / P0   [128,256) S1 / P1   [256,384) O0   [384,512) O1
// S = Q K^T lands in TMEM; the softmax warps read it (tcgen05.ld), write the
// bf16 probabilities P back over the first 64 columns of S (tcgen05.st), and
// the MMA warp computes O += P V with P as the tensor-memory A operand.  The
// two Q tiles ping-pong: while one warpgroup runs its softmax, the tensor core
// works on the other tile.  The running row max is only moved (and O
// rescaled) when it grows by more than 2^8 in probability units, so O is
// rarely touched by the softmax warps.
//
// Shared-memory tiles use the 128-byte swizzle: a 128 x 128 bf16 tile is two
// column halves of 64 channels (128 bytes per row); TMA writes them as 64-row
// boxes.  Q and K are K-major MMA operands; V is an MN-major operand.
// No TMA multicast is used anywhere.
#include <math.h>

#include "internal.h"

namespace mmdit {

namespace {

constexpr int kTileBytes = 128 * 128 * 2; // 32 KB: one 128 x 128 bf16 tile
constexpr int kHalfCol = 128 * 128;       // bytes of one 64-channel column half
constexpr int kBoxBytes = 64 * 128;       // one TMA box: 64 rows x 64 channels

// Kernel shape: QT Q tiles of 128 rows per CTA (one softmax warpgroup each)
// and an ST-slot K/V ring.  QT = 2 fills the SM (225 KB smem, 512 TMEM
// columns) and lets the two tiles ping-pong on the tensor core; QT = 1 with a
// 2-slot ring needs 105 KB and 256 columns, so two CTAs share an SM and hide
// each other's load and epilogue latency (used for short key sequences).
template <int QT, int ST>
struct Cfg {
  // QT softmax warpgroups + one warpgroup holding the TMA producer warp, the
  // MMA warp and two idle warps: the register file is handed out per
  // warpgroup, so the CTA is a whole number of them and setmaxnreg moves
  // registers from the producer/MMA warpgroup to the softmax warpgroups.
  static constexpr int kThreads = 128 * (QT + 1);
  static constexpr int kProducerWarp = 4 * QT;
  static constexpr int kMmaWarp = 4 * QT + 1;
  static constexpr int kStages = ST;
  // Paired ring (ST >= 4, one work item per CTA): key tile j's K and V share
  // one unit of two slots, one barrier that both TMA loads complete and one
  // release after the last PV of the tile, so the MMA thread waits and
  // commits once per key tile for the ring instead of twice (joint attention
  // 2 % faster).  Persistent CTAs, whose short items start while the ring
  // drains, and the 2-slot ring of the one-tile shape keep a slot (and a
  // barrier) per K or V tile.
  static constexpr bool kPairable = ST >= 4 && ST % 2 == 0;
  static constexpr int kRows = 128 * QT;  // query rows per CTA
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = QT * kTileBytes;
  // epilogue staging: per softmax warp 32 rows x kStageCols bf16 channels
  // (one row of kStageCols * 2 bytes per lane, 16-byte chunks swizzled as the
  // output map's 64- or 128-byte mode expects), so O leaves in whole 32-row
  // boxes instead of one row per lane; 1024-byte aligned like the tiles
  static constexpr int kStageCols = QT == 2 ? 64 : 32;
  static constexpr int kStageWarpBytes = 32 * kStageCols * 2;
  static constexpr int kStageOff = kKVOff + ST * kTileBytes;
  static constexpr int kBarOff = kStageOff + 4 * QT * kStageWarpBytes;
  static constexpr int kSmemBytes = kBarOff + 256 + 1024;  // + align slack
  static constexpr int kTmemCols = 256 * QT;               // S_t and O_t per tile
  static constexpr int kMinBlocks = QT == 1 ? 2 : 1;
  // Registers per thread: at launch 65,536 / (threads x CTAs per SM), rounded
  // down to 8; then the producer/MMA warpgroup drops to kRegsLow and the
  // softmax warpgroups rise to kRegsHigh, keeping
  // 128 * (QT * kRegsHigh + kRegsLow) <= kThreads * kRegsLaunch.
  static constexpr int kRegsLaunch = (65536 / (kThreads * kMinBlocks)) / 8 * 8;
  static constexpr int kRegsLow = QT == 2 ? 104 : 64;
  static constexpr int kRegsHigh = ((kThreads * kRegsLaunch / 128 - kRegsLow) / QT) / 8 * 8;
  static_assert(128 * (QT * kRegsHigh + kRegsLow) <= kThreads * kRegsLaunch, "register split");
};
constexpr float kRescaleLog2 = 8.0f;      // move the max only beyond a factor 2^8

// barrier indices (8 bytes each)
// Phases: Q, O and their "empty" barriers complete once per work item; S and
// P once per key tile; the ring barriers once per load.
enum {
  B_QFULL = 0,    // 2: Q tile landed (TMA)
  B_QREADY = 2,   // 2: Q tile rotated in place (fused RoPE), 128 arrivals
  B_KVFULL = 4,   // 4: ring slot landed (TMA)
  B_KVEMPTY = 8,  // 4: ring slot consumed (tcgen05.commit)
  B_SFULL = 12,   // 2: S tile ready in TMEM
  B_PFULL = 14,   // 2: P tile written to TMEM (128 arrivals)
  B_OFULL = 16,   // 2: last PV of the item done (O ready for the epilogue)
  B_QEMPTY = 18,  // 2: last QK of the item done (Q buffer reusable)
  B_OEMPTY = 20,  // 2: epilogue has read O out of TMEM (128 arrivals)
  B_MMADONE = 22, // 1: every MMA of the CTA done (teardown)
  B_PHALF = 23,   // 2: first 64 keys of the P tile written (128 arrivals)
  B_COUNT = 25
};

constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 128, 0, 0);  // Q, K: K-major
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 128, 0, 1);  // P (TMEM), V: MN-major

struct Work {
  int b, h, split, qtile;
  int q0;       // first query token of the CTA (row 0 of Q tile 0)
  int q_valid;  // valid query rows of the CTA (<= rows per CTA)
  int kv_lo, kv_hi;  // dense: key range
  int nkv;      // number of 128-row key tiles
  long long ubase;   // sparse: offset of the merged list
  int ucount;        // sparse: entries of the merged list (two per key tile)
  int g_first, g_nblk;
};


// Position of a work item in the mixed radix (query tile, split, head, batch),
// query tile fastest.
struct ItemPos {
  int qtile, split, h, b;
};

__device__ __forceinline__ ItemPos item_pos(const AttnProblem& pr, int item) {
  ItemPos p;
  p.qtile = item % pr.n_qtiles;
  int idx = item / pr.n_qtiles;
  p.split = idx % pr.n_splits;
  idx /= pr.n_splits;
  p.h = idx % pr.H;
  p.b = idx / pr.H;
  return p;
}

// The work items of this CTA: blockIdx.x and, in persistent launches, every
// gridDim.x-th item after it.  The stride's digits are found once, so a step
// is digit-wise addition with carry instead of four divisions; the walk ends
// when the batch digit reaches B (item >= n_qtiles * n_splits * H * B).  With
// an item order (sparse mode) the CTA walks positions blockIdx.x,
// blockIdx.x + gridDim.x, ... of that list instead, up to its length.
template <bool PERSIST, bool ORDER>
struct ItemWalk {
  ItemPos cur, stride;
  int pos, n_ord;  // ordered walk: position in pr.order and the list length
  __device__ __forceinline__ explicit ItemWalk(const AttnProblem& pr)
      : cur(item_pos(pr, (int)blockIdx.x)), stride(item_pos(pr, PERSIST ? (int)gridDim.x : 0)),
        pos((int)blockIdx.x), n_ord(0) {
    if (ORDER) {
      n_ord = *pr.n_order;
      if (pos < n_ord) cur = item_pos(pr, pr.order[pos]);
      else cur.b = pr.B;
    }
  }
  __device__ __forceinline__ bool more(const AttnProblem& pr) const { return cur.b < pr.B; }
  __device__ __forceinline__ void next(const AttnProblem& pr) {
    if (!PERSIST) {
      cur.b = pr.B;
      return;
    }
    if (ORDER) {
      pos += (int)gridDim.x;
      if (pos < n_ord) cur = item_pos(pr, pr.order[pos]);
      else cur.b = pr.B;
      return;
    }
    const int q = cur.qtile + stride.qtile;
    int cy = q >= pr.n_qtiles;
    cur.qtile = cy ? q - pr.n_qtiles : q;
    const int sp = cur.split + stride.split + cy;
    cy = sp >= pr.n_splits;
    cur.split = cy ? sp - pr.n_splits : sp;
    const int h = cur.h + stride.h + cy;
    cy = h >= pr.H;
    cur.h = cy ? h - pr.H : h;
    cur.b += stride.b + cy;
  }
};

// SPARSE: the block-sparse mode (query groups, merged key lists); the mode is
// a template parameter so that the dense launches carry none of its code.
template <bool SPARSE>
__device__ __forceinline__ Work decode_work(const AttnParams& P, const ItemPos& pos, int rows) {
  Work w;
  const AttnProblem& pr = P.prob;
  w.qtile = pos.qtile;
  w.split = pos.split;
  w.h = pos.h;
  w.b = pos.b;
  if (!SPARSE) {
    const int nq = pr.q_count != nullptr ? min(pr.Nq, pr.q_count[w.b]) : pr.Nq;
    w.q0 = w.qtile * rows;
    w.q_valid = min(rows, nq - w.q0);
    w.kv_lo = w.split * pr.kv_per_split;
    w.kv_hi = min(pr.Nkv, w.kv_lo + pr.kv_per_split);
    // an item past the valid rows of its batch item computes nothing
    w.nkv = (w.kv_hi > w.kv_lo && w.q_valid > 0) ? (w.kv_hi - w.kv_lo + 127) / 128 : 0;
    w.ubase = 0;
    w.ucount = 0;
    w.g_first = w.g_nblk = 0;
  } else {
    // a group index past the batch item's group count is an empty item
    const bool real = w.qtile < pr.n_groups[w.b];
    const int4 g = real ? pr.groups[(long long)w.b * pr.n_qtiles + w.qtile] : make_int4(0, 0, 0, 0);
    w.g_first = g.x;
    w.g_nblk = g.y;
    w.q0 = g.z;
    w.q_valid = g.w;
    w.kv_lo = 0;
    w.kv_hi = pr.Nkv;
    const long long lid = ((long long)w.b * pr.H + w.h) * pr.n_qtiles + w.qtile;
    w.ubase = lid * pr.ucap;
    w.ucount = real ? min(max(pr.ucnt[lid], 0), pr.ucap) : 0;
    w.nkv = (w.ucount + 1) / 2;
  }
  return w;
}

// Token start of the two 64-row halves of key tile j, and (sparse) the
// merged-list entries they come from.
template <bool SPARSE>
__device__ __forceinline__ void kv_tile(const AttnProblem& pr, const Work& w, int j, int ucount,
                                        int& s0, int& s1) {
  if (!SPARSE) {
    s0 = w.kv_lo + j * 128;
    s1 = s0 + 64;
  } else {
    s0 = (int)pr.ulist[w.ubase + 2 * j].x;
    s1 = (2 * j + 1 < ucount) ? (int)pr.ulist[w.ubase + 2 * j + 1].x : s0;  // else fully masked
  }
}

// Sparse mode: the query blocks (bits of the group) that selected any key
// block of key tile j, from the membership masks of its two list entries.
__device__ __forceinline__ uint32_t tile_members(const AttnProblem& pr, const Work& w, int j) {
  const uint4 e0 = pr.ulist[w.ubase + 2 * j];
  uint32_t m = e0.z | e0.w;
  if (2 * j + 1 < w.ucount) {
    const uint4 e1 = pr.ulist[w.ubase + 2 * j + 1];
    m |= e1.z | e1.w;
  }
  return (m | (m >> 16)) & 0xFFFFu;
}

// Sparse mode: for each 128-row Q tile of the group, the query blocks whose
// rows it holds (bit i = block i of the group).
template <int QT>
__device__ __forceinline__ void tile_blocks(const AttnProblem& pr, const Work& w,
                                            uint32_t (&qm)[QT]) {
  const int2* tb = pr.tab + (long long)w.b * pr.tab_cap + w.g_first;
  int acc = 0;
#pragma unroll
  for (int t = 0; t < QT; ++t) qm[t] = 0u;
  for (int i = 0; i < w.g_nblk; ++i) {
    const int len = tb[i].y;
#pragma unroll
    for (int t = 0; t < QT; ++t)
      if (acc < 128 * (t + 1) && acc + len > 128 * t) qm[t] |= 1u << i;
    acc += len;
  }
}

__device__ __forceinline__ void tma_tile(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                         int h, int b, int s0, int s1) {
  tma_load_4d(dst, map, bar, 0, h, s0, b);
  tma_load_4d(dst + kBoxBytes, map, bar, 0, h, s1, b);
  tma_load_4d(dst + kHalfCol, map, bar, 64, h, s0, b);
  tma_load_4d(dst + kHalfCol + kBoxBytes, map, bar, 64, h, s1, b);
}

// S_t = Q_t K^T : M=128 (query rows), N=128 (key rows), K=128 (channels) as
// 8 MMAs of K=16.  Both operands K-major, 128-byte swizzle; stepping K by 16
// channels moves the start address 32 bytes inside the swizzle atom, and the
// second 64-channel half lives kHalfCol bytes further.
__device__ __forceinline__ void mma_qk(uint32_t s_tmem, uint32_t q_smem, uint32_t k_smem) {
  // The descriptors' start-address field holds address >> 4, so stepping an
  // operand by `off` bytes adds off >> 4 to it (every address here is below
  // 256 KB: the 14-bit field does not wrap).  The eight MMAs go out in one
  // asm block, the first overwriting S and the rest accumulating; the
  // stepped descriptors are formed inside the block, two registers at a time.
  const uint64_t a = smem_desc_sw128(q_smem, 16, 1024);
  const uint64_t b = smem_desc_sw128(k_smem, 16, 1024);
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
      "add.s64 ta, %1, %4;\n\tadd.s64 tb, %2, %4;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ta, tb, %3, pt;\n\t"
      "add.s64 ta, ta, 2;\n\tadd.s64 tb, tb, 2;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ta, tb, %3, pt;\n\t"
      "add.s64 ta, ta, 2;\n\tadd.s64 tb, tb, 2;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ta, tb, %3, pt;\n\t"
      "add.s64 ta, ta, 2;\n\tadd.s64 tb, tb, 2;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ta, tb, %3, pt;\n\t}"
      ::"r"(s_tmem), "l"(a), "l"(b), "r"(kIdescQK), "l"((uint64_t)(kHalfCol >> 4)));
}

// O_t (+)= P_t V : M=128, N=128 (channels), K=128 (key rows).  P comes from
// tensor memory (16 bf16 per row = 8 columns per K step).  V is MN-major:
// 64-channel halves are LBO = kHalfCol apart, 8-row groups SBO = 1024 apart,
// and 16 key rows (one K step) are 2048 bytes.
template <int K0, int K1>
__device__ __forceinline__ void mma_pv_part(uint32_t o_tmem, uint32_t p_tmem, uint32_t v_smem,
                                            bool accumulate) {
  static_assert(K1 - K0 == 4, "four K steps per part");
  // V steps 16 key rows (2048 bytes: 128 in the descriptor) per K step; P
  // steps 8 TMEM columns.  The first MMA accumulates only if asked (or past
  // the first K step), the rest always.
  const uint64_t b = smem_desc_sw128(v_smem + K0 * 2048, kHalfCol, 1024);
  const uint32_t pa = p_tmem + K0 * 8;
  const uint32_t acc0 = (accumulate || K0 > 0) ? 1u : 0u;
  asm volatile(
      "{\n\t.reg .pred p0, pt;\n\t.reg .b64 tb;\n\t.reg .b32 ta;\n\t"
      "setp.ne.b32 p0, %4, 0;\n\t"
      "setp.eq.b32 pt, %4, %4;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p0;\n\t"
      "add.u32 ta, %1, 8;\n\tadd.s64 tb, %2, 128;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], tb, %3, pt;\n\t"
      "add.u32 ta, ta, 8;\n\tadd.s64 tb, tb, 128;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], tb, %3, pt;\n\t"
      "add.u32 ta, ta, 8;\n\tadd.s64 tb, tb, 128;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], tb, %3, pt;\n\t}"
      ::"r"(o_tmem), "r"(pa), "l"(b), "r"(kIdescPV), "r"(acc0));
}

// Rotate this thread's Q row (row r of the tile at q_smem) in place by the
// 3D RoPE angles of token `tok`.
__device__ void rope_row_smem(uint8_t* q_tile, int r, int tok, const DevLayout& L,
                              const RopeTab& tab) {
  float pt, ph, pw;
  token_position(L, tok, pt, ph, pw);
#pragma unroll 1
  for (int j = 0; j < 16; ++j) {  // 16 chunks of 8 channels
    const int half = j >> 3, jj = j & 7;
    uint4* p = reinterpret_cast<uint4*>(q_tile + half * kHalfCol + r * 128 +
                                        ((jj ^ (r & 7)) << 4));
    uint4 raw = *p;
    __nv_bfloat162* x = reinterpret_cast<__nv_bfloat162*>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int m = j * 4 + i;
      const float pos = m < tab.pt ? pt : (m < tab.ph ? ph : pw);
      float sn, cs;
      sincosf(pos * tab.omega[m], &sn, &cs);
      const float2 v = __bfloat1622float2(x[i]);
      x[i] = __float22bfloat162_rn(make_float2(v.x * cs - v.y * sn, v.x * sn + v.y * cs));
    }
    *p = raw;
  }
}

// PERSIST = false: one work item per CTA (grid = items; the loops below run
// once, so no cross-item state is live).  PERSIST = true: each CTA walks items
// blockIdx.x, blockIdx.x + gridDim.x, ... keeping TMEM and barriers alive, and
// the next item's Q load and QK overlap the current item's epilogue.
// ORDER: block-sparse mode, CTA i taking the i-th work item listed in
// pr.order (the items whose query group exists, in index order).
template <int QT, int ST, bool PERSIST, bool ORDER>
__global__ void __launch_bounds__(Cfg<QT, ST>::kThreads, Cfg<QT, ST>::kMinBlocks)
    attn_tc_kernel(const __grid_constant__ AttnParams P) {
  using C = Cfg<QT, ST>;
  constexpr int kStages = C::kStages;
  constexpr bool kPaired = C::kPairable && !PERSIST;
  constexpr int kUnits = kPaired ? ST / 2 : ST;  // ring units (barrier pairs)
  if (!PERSIST) {
    // a one-item CTA with nothing to compute or write (past the ordered
    // list, or past its batch item's valid query rows: the masked attention
    // sizes its grid for every video row) leaves before any set-up
    const ItemWalk<PERSIST, ORDER> w0(P.prob);
    if (!w0.more(P.prob)) return;
    if (!ORDER && decode_work<false>(P, w0.cur, C::kRows).q_valid <= 0) return;
  }
  constexpr int kQOff = C::kQOff;
  constexpr int kKVOff = C::kKVOff;
  constexpr int kBarOff = C::kBarOff;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bars = sbase + kBarOff;
  auto bar = [&](int i) { return bars + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kBarOff + 8 * B_COUNT);
  // sparse mode: per K/V ring slot, the query blocks that selected any key
  // block of the key tile loaded there (written by the producer before the
  // slot's TMA, read by the MMA warp after the slot's barrier completes)
  volatile uint32_t* slot_members = reinterpret_cast<volatile uint32_t*>(smem + kBarOff + 8 * B_COUNT + 16);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* err = P.err;
  const bool skip = *(volatile int*)err != 0;  // an earlier kernel timed out

  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(B_QFULL + t), 1);
      mbar_init(bar(B_QREADY + t), 128);
      mbar_init(bar(B_SFULL + t), 1);
      mbar_init(bar(B_PFULL + t), 128);
      mbar_init(bar(B_PHALF + t), 128);
      mbar_init(bar(B_OFULL + t), 1);
      mbar_init(bar(B_QEMPTY + t), 1);
      mbar_init(bar(B_OEMPTY + t), 128);
    }
    for (int u = 0; u < kUnits; ++u) {
      mbar_init(bar(B_KVFULL + u), 1);
      mbar_init(bar(B_KVEMPTY + u), 1);
    }
    mbar_init(bar(B_MMADONE), 1);
    fence_mbar_init();
  }
  if (warp == C::kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 4 * QT) {
    // producer / MMA warpgroup: give registers to the softmax warpgroups
    setmaxnreg_dec<C::kRegsLow>();
  if (warp == C::kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && !skip) {
      int last[kUnits];
#pragma unroll
      for (int i = 0; i < kUnits; ++i) last[i] = -1;
      bool ok = true;
      int ld = 0;  // ring units filled so far (all items)
      int it = 0;  // items of this CTA so far
      for (ItemWalk<PERSIST, ORDER> wk(P.prob); wk.more(P.prob) && ok; wk.next(P.prob), ++it) {
        const Work w = decode_work<ORDER>(P, wk.cur, C::kRows);
        const AttnProblem& pr = P.prob;
        if (it == 0) {
          tma_prefetch_desc(&pr.tmQ);
          tma_prefetch_desc(&pr.tmK);
          tma_prefetch_desc(&pr.tmV);
          if (!ORDER && pr.o != nullptr && pr.part_o == nullptr)
            tma_prefetch_desc(&pr.tmO);
        }
        for (int t = 0; t < QT && ok; ++t) {
          if (it > 0 && !(ok = mbar_wait(bar(B_QEMPTY + t), (it - 1) & 1, err))) break;
          mbar_expect_tx(bar(B_QFULL + t), kTileBytes);
          const int s0 = w.q0 + t * 128;
          tma_tile(sbase + kQOff + t * kTileBytes, &pr.tmQ, bar(B_QFULL + t), w.h, w.b, s0,
                   s0 + 64);
        }
        const int ucount = w.ucount;
        for (int j = 0; j < w.nkv && ok; ++j) {
          int s0, s1;
          kv_tile<ORDER>(pr, w, j, ucount, s0, s1);
          if (kPaired) {
            // K and V of key tile j into the two slots of one unit
            const int u = ld % kUnits;
            if (!(ok = mbar_wait(bar(B_KVEMPTY + u), ((ld / kUnits) & 1) ^ 1, err))) break;
            if (ORDER) slot_members[u] = tile_members(pr, w, j);
            mbar_expect_tx(bar(B_KVFULL + u), 2 * kTileBytes);
            tma_tile(sbase + kKVOff + 2 * u * kTileBytes, &pr.tmK, bar(B_KVFULL + u), w.h, w.b,
                     s0, s1);
            tma_tile(sbase + kKVOff + (2 * u + 1) * kTileBytes, &pr.tmV, bar(B_KVFULL + u), w.h,
                     w.b, s0, s1);
            last[u] = ld++;
          } else {
            for (int kind = 0; kind < 2; ++kind, ++ld) {
              const int slot = ld % kStages;
              if (!(ok = mbar_wait(bar(B_KVEMPTY + slot), ((ld / kStages) & 1) ^ 1, err))) break;
              if (ORDER && kind == 0) slot_members[slot] = tile_members(pr, w, j);
              mbar_expect_tx(bar(B_KVFULL + slot), kTileBytes);
              tma_tile(sbase + kKVOff + slot * kTileBytes, kind ? &pr.tmV : &pr.tmK,
                       bar(B_KVFULL + slot), w.h, w.b, s0, s1);
              last[slot] = ld;
            }
          }
        }
      }
      // every copy issued must land before the CTA's shared memory goes away
      if (it > 0)
        for (int t = 0; t < QT; ++t) mbar_wait(bar(B_QFULL + t), (it - 1) & 1, err);
      for (int u = 0; u < kUnits; ++u)
        if (last[u] >= 0) mbar_wait(bar(B_KVFULL + u), (last[u] / kUnits) & 1, err);
    }
  } else if (warp == C::kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    // Issue order per key tile j (t = Q tiles of the CTA):
    //   PV_t(j) then QK_t(j+1), tile after tile, so that P_t (which aliases S_t
    //   in TMEM) is consumed by PV_t before QK_t(j+1) overwrites S_t, and the
    //   completion of QK_t(j+1) also implies PV_t(j) is done.  PV_t(j) goes in
    //   two halves: keys 0..63 as soon as the softmax has written that half of
    //   P (p_half), keys 64..127 once the whole tile is written (p_full), so
    //   the tensor core starts while the second half is still being
    //   exponentiated.  Across items the first PV_t of an item waits until the
    //   epilogue has read O_t out.
    if (lane == 0 && !skip) {
      bool ok = true;
      int cs = 0;   // ring units consumed so far (all items)
      int pt = 0;   // key tiles processed so far (P barrier phases)
      int it = 0;
      for (ItemWalk<PERSIST, ORDER> wk(P.prob); wk.more(P.prob) && ok; wk.next(P.prob), ++it) {
        const Work w = decode_work<ORDER>(P, wk.cur, C::kRows);
        const AttnProblem& pr = P.prob;
        const int nkv = w.nkv;
        const int qbar = pr.rope_q ? B_QREADY : B_QFULL;
        for (int t = 0; t < QT && ok; ++t) ok = mbar_wait(bar(qbar + t), it & 1, err);
        if (!ok) break;
        // ring position of key tile j's K and V: a unit of two slots (paired
        // ring) or consecutive single slots
        auto k_unit = [&](int j) { return kPaired ? (cs + j) % kUnits : (cs + 2 * j) % kStages; };
        auto v_unit = [&](int j) { return kPaired ? (cs + j) % kUnits : (cs + 2 * j + 1) % kStages; };
        auto k_parity = [&](int j) { return (kPaired ? (cs + j) / kUnits : (cs + 2 * j) / kStages) & 1; };
        auto v_parity = [&](int j) { return (kPaired ? (cs + j) / kUnits : (cs + 2 * j + 1) / kStages) & 1; };
        auto k_smem_of = [&](int j) {
          return sbase + kKVOff + (kPaired ? 2 * k_unit(j) : k_unit(j)) * kTileBytes;
        };
        auto v_smem_of = [&](int j) {
          return sbase + kKVOff + (kPaired ? 2 * v_unit(j) + 1 : v_unit(j)) * kTileBytes;
        };
        if (nkv > 0) {
          // Sparse mode: a Q tile none of whose query blocks selected any key
          // block of key tile j skips that tile's QK and PV (the barriers
          // still complete, so both sides stay in phase); O_t is written by
          // its first PV without accumulation.
          uint32_t qm[QT];
          if (ORDER) tile_blocks<QT>(pr, w, qm);
          auto active = [&](uint32_t members, int t) { return !ORDER || (members & qm[t]) != 0u; };
          bool o_init[QT];
#pragma unroll
          for (int t = 0; t < QT; ++t) o_init[t] = false;
          // prologue: S_t = Q_t K_0^T for every tile
          const int s_k0 = k_unit(0);
          if (!(ok = mbar_wait(bar(B_KVFULL + s_k0), k_parity(0), err))) break;
          tc_fence_after();
          uint32_t mem_j = ORDER ? slot_members[s_k0] : ~0u;
#pragma unroll
          for (int t = 0; t < QT; ++t) {
            if (active(mem_j, t)) mma_qk(tmem + t * 128, sbase + kQOff + t * kTileBytes, k_smem_of(0));
            tc_commit(bar(B_SFULL + t));
            if (nkv == 1) tc_commit(bar(B_QEMPTY + t));
          }
          if (!kPaired) tc_commit(bar(B_KVEMPTY + s_k0));
          for (int j = 0; j < nkv && ok; ++j) {
            const int sv = v_unit(j), sk = k_unit(j + 1);
            const uint32_t v_smem = v_smem_of(j);
            const uint32_t k_smem = k_smem_of(j + 1);
            const bool more = j + 1 < nkv;
            uint32_t mem_next = ~0u;
            // paired ring: V(j) landed with K(j), whose unit was waited for
            if (!kPaired && !(ok = mbar_wait(bar(B_KVFULL + sv), v_parity(j), err))) break;
#pragma unroll
            for (int t = 0; t < QT; ++t) {
              const bool act = active(mem_j, t);
              if (!(ok = mbar_wait(bar(B_PHALF + t), (pt + j) & 1, err))) break;
              if (j == 0 && it > 0 && !(ok = mbar_wait(bar(B_OEMPTY + t), (it - 1) & 1, err)))
                break;
              tc_fence_after();
              if (act)
                mma_pv_part<0, 4>(tmem + QT * 128 + t * 128, tmem + t * 128, v_smem, o_init[t]);
              if (!(ok = mbar_wait(bar(B_PFULL + t), (pt + j) & 1, err))) break;
              tc_fence_after();
              if (act) {
                mma_pv_part<4, 8>(tmem + QT * 128 + t * 128, tmem + t * 128, v_smem, true);
                o_init[t] = true;
              }
              if (t == QT - 1) tc_commit(bar(B_KVEMPTY + sv));
              if (more) {
                if (t == 0) {
                  if (!(ok = mbar_wait(bar(B_KVFULL + sk), k_parity(j + 1), err))) break;
                  tc_fence_after();
                  if (ORDER) mem_next = slot_members[sk];
                }
                if (active(mem_next, t)) mma_qk(tmem + t * 128, sbase + kQOff + t * kTileBytes, k_smem);
                tc_commit(bar(B_SFULL + t));
                if (j + 2 == nkv) tc_commit(bar(B_QEMPTY + t));
                if (!kPaired && t == QT - 1) tc_commit(bar(B_KVEMPTY + sk));
              }
            }
            mem_j = mem_next;
          }
          cs += kPaired ? nkv : 2 * nkv;
          pt += nkv;
        } else {
          for (int t = 0; t < QT; ++t) {
            if (it > 0 && !(ok = mbar_wait(bar(B_OEMPTY + t), (it - 1) & 1, err))) break;
            tc_commit(bar(B_QEMPTY + t));
          }
        }
        for (int t = 0; t < QT; ++t) tc_commit(bar(B_OFULL + t));
      }
      tc_commit(bar(B_MMADONE));
      mbar_wait(bar(B_MMADONE), 0, err);
    }
  }  // warps 4*QT+2 and 4*QT+3 have no role
  } else {
    // ------------------------------------------------------------ softmax
    setmaxnreg_inc<C::kRegsHigh>();
    const int t = warp >> 2;                  // Q tile of this warpgroup
    const int r = (warp & 3) * 32 + lane;     // row inside the tile == TMEM lane
    const int row = t * 128 + r;              // row inside the CTA's rows
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t s_addr = tmem + lane_off + t * 128;
    const uint32_t o_addr = tmem + lane_off + QT * 128 + t * 128;
    const float sl2 = P.scale_log2;
    const float thresh = kRescaleLog2 / sl2;  // in raw score units

    const uint64_t sl2x2 = pack_f32x2(sl2, sl2);
    bool ok = !skip;
    int st = 0;  // S tiles consumed so far (all items)
    int it = 0;
    for (ItemWalk<PERSIST, ORDER> wk(P.prob); wk.more(P.prob) && ok; wk.next(P.prob), ++it) {
      const Work w = decode_work<ORDER>(P, wk.cur, C::kRows);
      const AttnProblem& pr = P.prob;
      const int nkv = w.nkv;

      if (pr.rope_q) {
        ok = mbar_wait(bar(B_QFULL + t), it & 1, err);
        if (ok) {
          rope_row_smem(smem + kQOff + t * kTileBytes, r, w.q0 + row, P.layout, P.rope);
          fence_proxy_async_smem();
        }
        mbar_arrive(bar(B_QREADY + t));
      }

      // sparse mode: which query block of the group this row belongs to
      int qb = 0;
      int ucount = 0;
      if (ORDER) {
        int acc = 0;
        qb = -1;  // rows past the group: member of nothing
        const int2* tb = pr.tab + (long long)w.b * pr.tab_cap + w.g_first;
        for (int i = 0; i < w.g_nblk; ++i) {
          const int blen = tb[i].y;
          if (row < acc + blen) {
            qb = i;
            break;
          }
          acc += blen;
        }
        ucount = w.ucount;
      }
      // sparse mode: the query blocks of this warpgroup's Q tile (a key tile
      // none of them selected is skipped by the whole warpgroup, as by the
      // MMA warp)
      uint32_t tile_qm = ~0u;
      if (ORDER) {
        uint32_t qm[QT];
        tile_blocks<QT>(pr, w, qm);
        tile_qm = qm[t];
      }
      bool o_written = false;  // a PV of this item has written O_t

      float m_used = -INFINITY, l = 0.f;
      for (int j = 0; j < nkv; ++j, ++st) {
        // valid key columns of each 64-row half of this tile for this row
        // (independent of S, so computed before waiting for it)
        int len0, len1;
        uint32_t seg0 = 0xFu, seg1 = 0xFu;  // valid 16-row segments of each half
        if (!ORDER) {
          const int s0 = w.kv_lo + j * 128;
          len0 = max(0, min(64, w.kv_hi - s0));
          len1 = max(0, min(64, w.kv_hi - s0 - 64));
        } else {
          const uint4 e0 = pr.ulist[w.ubase + 2 * j];
          const uint4 e1 = (2 * j + 1 < ucount) ? pr.ulist[w.ubase + 2 * j + 1]
                                                : make_uint4(0u, 0u, 0u, 0u);
          len0 = (int)e0.y;
          len1 = (int)e1.y;
          // this row's query block (0..15) in each segment's membership mask;
          // rows past the group (qb < 0) are members of nothing
          if (qb >= 0) {
            seg0 = ((e0.z >> qb) & 1u) | (((e0.z >> (16 + qb)) & 1u) << 1) |
                   (((e0.w >> qb) & 1u) << 2) | (((e0.w >> (16 + qb)) & 1u) << 3);
            seg1 = ((e1.z >> qb) & 1u) | (((e1.z >> (16 + qb)) & 1u) << 1) |
                   (((e1.w >> qb) & 1u) << 2) | (((e1.w >> (16 + qb)) & 1u) << 3);
          } else {
            seg0 = seg1 = 0u;
          }
        }
        bool tile_on = true;
        if (ORDER) {
          const uint4 f0 = pr.ulist[w.ubase + 2 * j];
          uint32_t mm = f0.z | f0.w;
          if (2 * j + 1 < ucount) {
            const uint4 f1 = pr.ulist[w.ubase + 2 * j + 1];
            mm |= f1.z | f1.w;
          }
          tile_on = (((mm | (mm >> 16)) & 0xFFFFu) & tile_qm) != 0u;
        }
        ok = ok && mbar_wait(bar(B_SFULL + t), st & 1, err);
        if (__any_sync(0xffffffffu, !ok)) {
          ok = false;
          break;
        }
        if (!tile_on) {
          // no QK was issued for this tile: release both P barriers at once
          tc_fence_before();
          mbar_arrive(bar(B_PHALF + t));
          mbar_arrive(bar(B_PFULL + t));
          continue;
        }
        __syncwarp();
        tc_fence_after();
        float s[128];
        {
          uint32_t v0[32], v1[32], v2[32], v3[32];
          tmem_ld32(s_addr, v0);
          tmem_ld32(s_addr + 32, v1);
          tmem_ld32(s_addr + 64, v2);
          tmem_ld32(s_addr + 96, v3);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            s[i] = __uint_as_float(v0[i]);
            s[32 + i] = __uint_as_float(v1[i]);
            s[64 + i] = __uint_as_float(v2[i]);
            s[96 + i] = __uint_as_float(v3[i]);
          }
        }
        const bool masked = len0 < 64 || len1 < 64 || seg0 != 0xFu || seg1 != 0xFu;
        if (masked) {
          // per 16-column segment: the valid columns are a prefix (the key
          // run's length cuts at most one segment per half; a segment whose
          // membership bit is clear has none), so a full segment costs one
          // comparison and only a cut or cleared one touches its columns
#pragma unroll
          for (int g = 0; g < 8; ++g) {
            const uint32_t segm = g < 4 ? seg0 : seg1;
            const int len = g < 4 ? len0 : len1;
            const int base = (g & 3) * 16;
            const int lim = ((segm >> (g & 3)) & 1u) ? min(max(len - base, 0), 16) : 0;
            if (lim < 16) {
#pragma unroll
              for (int i = 0; i < 16; ++i)
                if (i >= lim) s[(g >> 2) * 64 + base + i] = -INFINITY;
            }
          }
        }
        const float mt = row_max128(s);
        const bool grow = mt > m_used + thresh || (m_used == -INFINITY && mt > -INFINITY);
        float alpha = 1.f;
        if (grow) {
          alpha = (m_used == -INFINITY) ? 0.f : ex2_approx((m_used - mt) * sl2);
          m_used = mt;
          l *= alpha;
        }
        if (o_written && __any_sync(0xffffffffu, grow)) {
          // rescale the running O of this row (previous PV is complete: it was
          // issued before the QK whose completion released this S tile)
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t v[32];
            tmem_ld32(o_addr + c * 32, v);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * alpha);
            tmem_st32(o_addr + c * 32, v);
          }
          tmem_wait_st();
        }
        const float mref = (m_used == -INFINITY) ? 0.f : m_used * sl2;
        const uint64_t nm2 = pack_f32x2(-mref, -mref);
        // exponentials on the MUFU (ex2), arguments formed two at a time
        uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const uint64_t x2 = ffma_f32x2(pack_f32x2(s[c * 32 + 2 * i], s[c * 32 + 2 * i + 1]),
                                           sl2x2, nm2);
            float p0, p1;
            unpack_f32x2(x2, p0, p1);
            p0 = ex2_approx(p0);
            p1 = ex2_approx(p1);
            pk[i] = pack_bf16x2(p0, p1);
            acc[i & 3] = add_f32x2(acc[i & 3], pack_f32x2(p0, p1));
          }
          tmem_st16(s_addr + c * 16, pk);  // P: 2 bf16 per column
          if (c == 1) {  // keys 0..63 of P written: the first half of PV may start
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(B_PHALF + t));
          }
        }
        tmem_wait_st();
        {
          float a0, a1, b0, b1;
          unpack_f32x2(add_f32x2(acc[0], acc[1]), a0, a1);
          unpack_f32x2(add_f32x2(acc[2], acc[3]), b0, b1);
          l += (a0 + a1) + (b0 + b1);
        }
        tc_fence_before();
        mbar_arrive(bar(B_PFULL + t));
        o_written = true;
      }

      // ---------------------------------------------------------- epilogue
      ok = ok && mbar_wait(bar(B_OFULL + t), it & 1, err);
      if (__any_sync(0xffffffffu, !ok)) {
        ok = false;
        break;
      }
      __syncwarp();
      tc_fence_after();
      const bool valid_row = row < w.q_valid;
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const int qrow = w.q0 + row;
      // O row into registers with one TMEM round trip, then hand TMEM back to
      // the MMA warp before any global store (the next item's first PV may
      // overwrite O while this warpgroup stores)
      uint32_t o0[32], o1[32], o2[32], o3[32];
      if (o_written) {
        tmem_ld32(o_addr, o0);
        tmem_ld32(o_addr + 32, o1);
        tmem_ld32(o_addr + 64, o2);
        tmem_ld32(o_addr + 96, o3);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) o0[i] = o1[i] = o2[i] = o3[i] = 0u;
      }
      tc_fence_before();
      mbar_arrive(bar(B_OEMPTY + t));
      auto ov = [&](int c) -> uint32_t {  // column c of this row (compile-time c)
        return c < 32 ? o0[c] : c < 64 ? o1[c - 32] : c < 96 ? o2[c - 64] : o3[c - 96];
      };
      if (pr.part_o != nullptr) {
        // split-KV partial: unnormalised O, running max (log2 units) and sum
        const long long prow =
            (((long long)w.split * pr.B + w.b) * pr.H + w.h) * (long long)(pr.n_qtiles * C::kRows) +
            (long long)w.qtile * C::kRows + row;
        float* dst = pr.part_o + prow * 128;
        if (valid_row) {
#pragma unroll
          for (int i = 0; i < 128; i += 4)
            *reinterpret_cast<float4*>(dst + i) =
                make_float4(__uint_as_float(ov(i)), __uint_as_float(ov(i + 1)),
                            __uint_as_float(ov(i + 2)), __uint_as_float(ov(i + 3)));
          pr.part_ml[prow * 2 + 0] = (m_used == -INFINITY) ? -INFINITY : m_used * sl2;
          pr.part_ml[prow * 2 + 1] = l;
        }
      } else if (!ORDER) {
        if (pr.row_sq != nullptr && valid_row) {
          // squared L2 norm of the normalised row (the A->V output norms
          // that guide the content-adaptive block shapes)
          float ss = 0.f;
#pragma unroll
          for (int c = 0; c < 128; ++c) {
            const float x = __uint_as_float(ov(c)) * inv;
            ss = fmaf(x, x, ss);
          }
          pr.row_sq[((long long)w.b * pr.Nq + qrow) * pr.H + w.h] = ss;
        }
        // normalised bf16 O through the TMA engine: each round packs
        // kStageCols channels of the warp's 32 rows into the warp's staging
        // buffer and one lane issues a bulk tensor store of that box; the
        // buffer is rewritten only once the previous store has read it.  Rows
        // past the end of the sequence lie outside the map and are not written.
        constexpr int SC = C::kStageCols;
        constexpr int CH = SC / 8;  // 16-byte chunks per staged row
        const int wrow = t * 128 + (warp & 3) * 32;  // first row of this warp inside the CTA
        if (wrow < w.q_valid) {
          uint8_t* stg = smem + C::kStageOff + warp * C::kStageWarpBytes;
          const int sw = ((lane * SC * 2) >> 7) & (CH - 1);  // swizzle of this lane's row
#pragma unroll
          for (int r = 0; r < 128 / SC; ++r) {
            if (lane == 0) bulk_wait_read<0>();
            __syncwarp();
#pragma unroll
            for (int chunk = 0; chunk < CH; ++chunk) {
              const int c0 = r * SC + chunk * 8;
              uint4 pk;
              pk.x = pack_bf16x2(__uint_as_float(ov(c0 + 0)) * inv, __uint_as_float(ov(c0 + 1)) * inv);
              pk.y = pack_bf16x2(__uint_as_float(ov(c0 + 2)) * inv, __uint_as_float(ov(c0 + 3)) * inv);
              pk.z = pack_bf16x2(__uint_as_float(ov(c0 + 4)) * inv, __uint_as_float(ov(c0 + 5)) * inv);
              pk.w = pack_bf16x2(__uint_as_float(ov(c0 + 6)) * inv, __uint_as_float(ov(c0 + 7)) * inv);
              *reinterpret_cast<uint4*>(stg + lane * (SC * 2) + ((chunk ^ sw) << 4)) = pk;
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_4d(&pr.tmO, smem_u32(stg), r * SC, w.h, w.q0 + wrow, w.b);
              bulk_commit();
            }
          }
        }
        if (pr.lse != nullptr && valid_row) {
          const float mref = (m_used == -INFINITY) ? 0.f : m_used * sl2;
          pr.lse[((long long)w.b * pr.H + w.h) * pr.Nq + qrow] =
              l > 0.f ? (mref + log2f(l)) * 0.69314718055994531f : -INFINITY;
        }
      } else {
        // normalised bf16 O (sparse mode, where the rows past a query group
        // belong to the next group): each round stages kStageCols channels of the
        // warp's 32 rows in shared memory (16-byte chunks XOR-swizzled by row,
        // conflict-free both ways), then writes them back so that a group of
        // lanes covers one row's contiguous bytes
        constexpr int SC = C::kStageCols;
        constexpr int CH = SC / 8;  // 16-byte chunks per staged row
        uint8_t* stage = smem + C::kStageOff + warp * C::kStageWarpBytes;
        const int wrow0 = (warp & 3) * 32;  // first row of this warp inside the tile
#pragma unroll
        for (int r = 0; r < 128 / SC; ++r) {
#pragma unroll
          for (int chunk = 0; chunk < CH; ++chunk) {
            const int c0 = r * SC + chunk * 8;
            uint4 pk;
            pk.x = pack_bf16x2(__uint_as_float(ov(c0 + 0)) * inv, __uint_as_float(ov(c0 + 1)) * inv);
            pk.y = pack_bf16x2(__uint_as_float(ov(c0 + 2)) * inv, __uint_as_float(ov(c0 + 3)) * inv);
            pk.z = pack_bf16x2(__uint_as_float(ov(c0 + 4)) * inv, __uint_as_float(ov(c0 + 5)) * inv);
            pk.w = pack_bf16x2(__uint_as_float(ov(c0 + 6)) * inv, __uint_as_float(ov(c0 + 7)) * inv);
            *reinterpret_cast<uint4*>(stage + lane * (SC * 2) + ((chunk ^ (lane % CH)) << 4)) = pk;
          }
          __syncwarp();
          constexpr int RPI = 32 / CH;  // rows per store instruction
#pragma unroll
          for (int i = 0; i < 32 / RPI; ++i) {
            const int srow = i * RPI + lane / CH, chunk = lane % CH;
            const uint4 pk = *reinterpret_cast<const uint4*>(stage + srow * (SC * 2) +
                                                             ((chunk ^ (srow % CH)) << 4));
            const int trow = t * 128 + wrow0 + srow;  // row inside the CTA
            if (trow < w.q_valid) {
              __nv_bfloat16* dst = pr.o + (long long)w.b * pr.o_sb +
                                   (long long)(w.q0 + trow) * pr.o_st + (long long)w.h * 128 +
                                   r * SC + chunk * 8;
              *reinterpret_cast<uint4*>(dst) = pk;
            }
          }
          __syncwarp();
        }
        if (pr.lse != nullptr && valid_row) {
          const float mref = (m_used == -INFINITY) ? 0.f : m_used * sl2;
          pr.lse[((long long)w.b * pr.H + w.h) * pr.Nq + qrow] =
              l > 0.f ? (mref + log2f(l)) * 0.69314718055994531f : -INFINITY;
        }
      }
    }
  }

  // ------------------------------------------------------------ teardown
  // output stores issued from shared memory complete before the CTA exits
  bulk_wait<0>();
  tc_fence_before();
  __syncthreads();
  if (warp == C::kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// Merge split-KV partials: O = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s.
// One warp per query row; lane l owns channels 4l..4l+3 (float4 loads of every
// split's 512-byte partial row), split weights computed once per row.
__global__ void __launch_bounds__(256) split_combine_kernel(const float* __restrict__ part_o,
                                                            const float* __restrict__ part_ml,
                                                            __nv_bfloat16* o, long long o_st,
                                                            long long o_sb, int n_splits, int B,
                                                            int H, int Nq, int Nq_pad) {
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);  // over B * H * Nq
  if (row >= (long long)B * H * Nq) return;
  const int q = (int)(row % Nq);
  const int h = (int)((row / Nq) % H);
  const int b = (int)(row / ((long long)Nq * H));
  const long long stride = (long long)B * H * Nq_pad;  // rows between splits
  const long long r0 = ((long long)b * H + h) * Nq_pad + q;
  float M = -INFINITY;
  for (int s = lane; s < n_splits; s += 32) M = fmaxf(M, part_ml[(r0 + s * stride) * 2]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  float L = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s = 0; s < n_splits; ++s) {
    const long long pr = r0 + s * stride;
    const float m = part_ml[pr * 2];
    if (m == -INFINITY) continue;
    const float f = exp2f(m - M);
    L += f * part_ml[pr * 2 + 1];
    const float4 v = *reinterpret_cast<const float4*>(part_o + pr * 128 + lane * 4);
    acc.x += f * v.x;
    acc.y += f * v.y;
    acc.z += f * v.z;
    acc.w += f * v.w;
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  uint2 pk;
  pk.x = pack_bf16x2(acc.x * inv, acc.y * inv);
  pk.y = pack_bf16x2(acc.z * inv, acc.w * inv);
  *reinterpret_cast<uint2*>(o + (long long)b * o_sb + (long long)q * o_st + (long long)h * 128 +
                            lane * 4) = pk;
}

template <int QT, int ST, bool PERSIST, bool ORDER = false>
cudaError_t launch_shape(const AttnParams& p, cudaStream_t s) {
  using C = Cfg<QT, ST>;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  // the dynamic shared-memory limit is a per-device function attribute
  e = once_per_device(dev, [] {
    return cudaFuncSetAttribute(attn_tc_kernel<QT, ST, PERSIST, ORDER>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  });
  if (e != cudaSuccess) return e;
  const int items = p.prob.ctas;
  if (items == 0) return cudaSuccess;
  int grid = items;
  if (PERSIST) {
    // one CTA per resident slot; each CTA walks items blockIdx.x + k*gridDim.x
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    grid = std::min(items, sms * C::kMinBlocks);
  }
  attn_tc_kernel<QT, ST, PERSIST, ORDER><<<grid, C::kThreads, C::kSmemBytes, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

int attn_store_cols(int q_tiles) {
  return q_tiles == 1 ? Cfg<1, 2>::kStageCols : Cfg<2, 4>::kStageCols;
}

int attn_rows_per_cta(int q_tiles) { return 128 * q_tiles; }

cudaError_t launch_attn_tc(const AttnParams& p, cudaStream_t s) {
  if (p.prob.order != nullptr) {
    // block-sparse attention over a list of work items: one CTA per listed
    // item (grid = the list's capacity; CTAs past its length exit at once)
    if (p.q_tiles != 2 || p.persistent) return cudaErrorInvalidValue;
    return launch_shape<2, 4, false, true>(p, s);
  }
  if (p.q_tiles == 1)  // one-tile CTAs are always persistent (short key sequences)
    return p.persistent ? launch_shape<1, 2, true>(p, s) : cudaErrorInvalidValue;
  return p.persistent ? launch_shape<2, 4, true>(p, s) : launch_shape<2, 4, false>(p, s);
}

cudaError_t launch_split_combine(const float* part_o, const float* part_ml, __nv_bfloat16* o,
                                 long long o_st, long long o_sb, int n_splits, int B, int H,
                                 int Nq, int Nq_pad, cudaStream_t s) {
  const long long rows = (long long)B * H * Nq;
  if (rows == 0) return cudaSuccess;
  split_combine_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(part_o, part_ml, o, o_st, o_sb,
                                                                 n_splits, B, H, Nq, Nq_pad);
  return cudaGetLastError();
}

}  // namespace mmdit
