// lod_prefill_tc.cu -- grouped chunked prefill of LoD attention on tcgen05
// tensor cores (bf16 caches, d = 128).
//
// What each query row computes is "Level of Detail Attention", How It Works
// paragraphs 2-3 (the same as lod_decode).  How the rows are organised
// follows "Coarse Semantic Blocks for Efficient Training-Free Sparse
// Attention", Abstract: in prefill, the queries that pick the same block are
// handled together, which keeps prefill fast.  Here the block is an index
// group, and the rows that opened it share one dense tensor-core tile.  Per
// wave of query chunks:
//
//  A  pf_scan_kernel   one CTA per 128 query rows of one KV head (128/g
//                      positions x g heads, all in one query chunk, so they
//                      share one visible index).  S = Q K^T on the tensor
//                      cores against every visible group summary, the sinks
//                      and the causal block window (keys on N), one online
//                      softmax per row (group logits carry + ln count), and
//                      O += P V on the tensor cores; each row's top-G groups
//                      are kept in registers by two selection warpgroups.
//                      The epilogue stores the row state, the top-G groups
//                      with the weights of their coarse terms, and counts
//                      the (row, group) pairs of every group.
//  plan, scatter       counting sort of the pairs by (KV head, group) and
//                      the work items (one group's pairs, up to kItemRows).
//  B  pf_pair_kernel   per work item the group's member keys and values and
//                      its page summaries are staged once.  For tiles of 128
//                      pairs (the rows that opened the group) S = Q K_g^T
//                      and Sp = Q pK^T score every member and page summary;
//                      each row opens its top_pages pages, and O = P [V_g; pV]
//                      adds the opened members exactly and the unopened pages
//                      as coarse entries (page mean value, logit + ln count)
//                      in one MMA chain.  The pair's normalised partial
//                      (log-sum-exp, bf16 output) is stored.
//  merge               per row: the opened groups' coarse terms leave the
//                      row state (finer entries replace them in B), then the
//                      state and its pairs' partials form one softmax; out
//                      and lse.
//
// Softmax arithmetic is in log2 units (logit * log2 e) with ex2 on the SFU.
// Removing the opened groups' coarse terms after the fact is numerically
// safe for the reason given in lod_attend.cu: the entries that replace a
// group carry at least its mass (n exp(q.mean k) <= sum exp(q.k)).
#include <cudaTypedefs.h>

#include "lod_internal.cuh"
#include "lod_tc.cuh"

namespace lod {

namespace {

constexpr int D = 128;
constexpr int kRows = 128;                      // query rows (or pairs) per tile: MMA M
constexpr uint32_t kTileBytes = 128 * D * 2;    // one 128 x 128 bf16 operand tile
constexpr uint32_t kHalf = kTileBytes / 2;      // one 64-column half of it
constexpr float kTau2 = 12.f;                   // weights reach at most 2^kTau2 before the reference max moves
constexpr int kStateStride = 132;               // floats per row state: m, l, -, -, acc[128]
constexpr int kSmallN = 112;  // pair kernel: groups up to this size run two CTAs per SM (members + 16 page columns fit 128)

__device__ __forceinline__ uint32_t sw_off(int row, int chunk16) {  // 16-byte chunk of a 128B-swizzled row
  return (uint32_t)(row * 128 + (((chunk16 & 7) ^ (row & 7)) << 4));
}

// ================================================================== phase A

// Warpgroups of the scan: 0 (warps 0-3) warp 0 TMA copies, warp 1 MMA
// issue; 1 (warps 4-7) softmax; 2 and 3 (warps 8-15) the top-G groups of
// key columns [0, 64) and [64, 128) of every group tile, and (group 2) the
// epilogue.  Registers move from warpgroup 0 to the others:
// 128 x (40 + 200 + 136 + 136) = 65536, the register file.
constexpr int kThreadsA = 512;
constexpr int kRegCtl = 40, kRegSoft = 200, kRegSel = 136;
constexpr int kCandCap = 28;     // buffered top-G candidates per row and column half
constexpr int kBarLncA = 1;      // named barrier of the softmax warps
constexpr int kBarEpiA = 2;      // named barrier of warpgroups 1 and 2 (hand-over of the softmax state)
constexpr int kBarSelA = 3;      // named barrier of warpgroups 2 and 3 (merge of the two column halves)
constexpr int kBarEndA = 4;      // named barrier of warpgroups 0-2 before TMEM is released

// Tensor memory of the scan: S double-buffered in columns [0, 256), O in
// [256, 384), the weights P (bf16 pairs, MMA 2's A operand) double-buffered
// in [384, 512), so the softmax of tile i + 1 does not wait for MMA 2 of
// tile i.
constexpr uint32_t kColO = 256, kColP = 384;

struct SmemA {
  static constexpr size_t off_K = 0;                          // [2 stages][2 halves][128][128 B]
  static constexpr size_t off_V = off_K + 2 * kTileBytes;     // [2 stages]
  static constexpr size_t off_Q = off_V + 2 * kTileBytes;     // the query tile [2 halves][128][128 B]
  static constexpr size_t off_cand = off_Q + kTileBytes;      // float2 [2][128][kCandCap + 1] (+1: odd row stride)
  static constexpr size_t off_meta = off_cand + 2 * 128 * (kCandCap + 1) * 8;  // int [2][128]
  static constexpr size_t off_lnc = off_meta + 2 * 128 * 4;   // float [2][128]
  static constexpr size_t off_ml = off_lnc + 2 * 128 * 4;   // float2 [128] softmax state handed over
  static constexpr int kBars = 20;
  static constexpr size_t off_bar = off_ml + 128 * 8;
  static constexpr size_t off_misc = off_bar + 8 * kBars;     // tmem slot, abort flag
  static constexpr size_t bytes = off_misc + 16 + 1024;
  static_assert(bytes <= 227 * 1024, "shared memory of one CTA");
};

// Insert (v, id) into the descending list (s, ix) of GM entries: every entry
// from the first one v beats moves down by one place.  Ties keep the earlier
// entry first (ids arrive in increasing order, so the lower id wins).  A
// list of G < GM entries occupies the last G slots below GM - G sentinels of
// +inf, so that its G-th best is always s[GM - 1] (a runtime index into a
// register array would move the list to local memory).
template <int GM>
__device__ __forceinline__ void topk_insert(float (&s)[GM], int (&ix)[GM], float v, int id) {
  bool act = false;
  float cs = v;
  int ci = id;
#pragma unroll
  for (int k = 0; k < GM; ++k) {  // selects only: the list stays in registers
    act = act || (v > s[k]);
    const float ns = act ? cs : s[k];
    const int ni = act ? ci : ix[k];
    cs = act ? s[k] : cs;
    ci = act ? ix[k] : ci;
    s[k] = ns;
    ix[k] = ni;
  }
}

// Insert (v, id) by the full ranking (score desc, id asc), for entries that
// do not arrive in id order.
template <int GM>
__device__ __forceinline__ void topk_insert_ranked(float (&s)[GM], int (&ix)[GM], float v, int id) {
  bool act = false;
  float cs = v;
  int ci = id;
#pragma unroll
  for (int k = 0; k < GM; ++k) {
    act = act || v > s[k] || (v == s[k] && (unsigned)id < (unsigned)ix[k]);
    const float ns = act ? cs : s[k];
    const int ni = act ? ci : ix[k];
    cs = act ? s[k] : cs;
    ci = act ? ix[k] : ci;
    s[k] = ns;
    ix[k] = ni;
  }
}

// Store 16 consecutive 32-bit columns of this thread's TMEM lane, without
// waiting (tmem_st_wait() before an MMA or another thread reads them).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15, %16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

// Wait until this thread's earlier TMEM stores have completed.
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Store (x, y) to shared memory at p when c holds (a predicated store: a
// miss costs an issue slot but no shared-memory bandwidth).
__device__ __forceinline__ void sts_f2_if(float2* p, float x, float y, bool c) {
  asm volatile(
      "{\n .reg .pred q;\n setp.ne.b32 q, %3, 0;\n @q st.shared.v2.f32 [%0], {%1, %2};\n}" ::"r"(smem_u32(p)),
      "f"(x), "f"(y), "r"((int)c)
      : "memory");
}

template <int N>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// Merge a row's buffered candidates (ascending ids: ties keep the earlier
// one) into its sorted list; the whole warp calls it.
template <int GM>
__device__ __forceinline__ void topk_merge(float (&s)[GM], int (&ix)[GM], float& thr, int& n, const float2* buf) {
  const int nmax = (int)__reduce_max_sync(0xffffffffu, (unsigned)n);
  for (int j0 = 0; j0 < nmax; j0 += 4) {
    float2 cv[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) cv[q] = j0 + q < n ? buf[j0 + q] : make_float2(-INFINITY, 0.f);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (cv[q].x > thr) {
        topk_insert<GM>(s, ix, cv[q].x, __float_as_int(cv[q].y));
        thr = s[GM - 1];
      }
    }
  }
  n = 0;
  __syncwarp();
}

template <int GM>
__global__ void __launch_bounds__(kThreadsA, 1)
    pf_scan_kernel(const __grid_constant__ TcMaps maps, const __grid_constant__ PrefillArgs a) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                       ~uintptr_t(1023));
  unsigned char* Kring = sm + SmemA::off_K;
  unsigned char* Vring = sm + SmemA::off_V;
  unsigned char* Qs = sm + SmemA::off_Q;
  float2* cand_s = reinterpret_cast<float2*>(sm + SmemA::off_cand);
  int* meta_s = reinterpret_cast<int*>(sm + SmemA::off_meta);
  float* lnc_s = reinterpret_cast<float*>(sm + SmemA::off_lnc);
  float2* ml_s = reinterpret_cast<float2*>(sm + SmemA::off_ml);
  uint64_t* kfull = reinterpret_cast<uint64_t*>(sm + SmemA::off_bar);
  uint64_t* kempty = kfull + 2;
  uint64_t* vfull = kempty + 2;
  uint64_t* vempty = vfull + 2;
  uint64_t* s_full = vempty + 2;
  uint64_t* s_free = s_full + 2;
  uint64_t* p_full = s_free + 2;  // [2]: weights of tile i written (buffer i & 1)
  uint64_t* o_done = p_full + 2;  // [2]: MMA 2 of tile i complete
  uint64_t* fin = o_done + 2;
  uint64_t* lnc_ready = fin + 1;  // [2]: ln counts of a group tile written
  uint64_t* q_ready = lnc_ready + 2;  // the query tile is in shared memory
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + SmemA::off_misc);
  volatile int* abort_s = reinterpret_cast<volatile int*>(sm + SmemA::off_misc + 4);

  // ---- the tile: heaviest (latest positions) first
  const int RP = kRows / a.g;                                // positions per tile
  const int64_t npos = a.w_hi - a.w_lo;
  const int64_t nblk = (npos + RP - 1) / RP;
  const int64_t units = (int64_t)a.B * a.Hkv;
  const int64_t blk = nblk - 1 - (int64_t)blockIdx.x / units;
  const int64_t u = (int64_t)blockIdx.x % units;             // b * Hkv + kvh
  const int b = (int)(u / a.Hkv), kvh = (int)(u % a.Hkv);
  const int64_t pos0 = a.w_lo + blk * RP;                    // first q position of the tile
  const int64_t pos_end = (pos0 + RP < a.w_hi) ? pos0 + RP : a.w_hi;
  const int64_t t0 = a.q_begin + pos0, t_max = a.q_begin + pos_end - 1;
  const int64_t bt = t0 / kChunk;                            // the tile's query chunk
  const int64_t nw = a.window / kChunk;
  const int64_t wb = bt - nw + 1 > 0 ? bt - nw + 1 : 0;
  const int64_t ws = wb * kChunk;                            // window start
  const int64_t G_vis = wb * a.k;
  const int64_t nsk = a.sinks < ws ? a.sinks : ws;
  const int gt = (int)((G_vis + 127) / 128);
  const int st_ = (int)((nsk + 127) / 128);
  const int ntile = gt + st_ + (int)((t_max - ws + 1 + 127) / 128);
  const int64_t Gcap = a.Cmax * a.k;
  const int64_t grow0 = u * Gcap;                            // this unit's first group row

  if (warp == 0 && lane == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&kfull[i], 1);
      mbar_init(&kempty[i], 1);
      mbar_init(&vfull[i], 1 + 32);
      mbar_init(&vempty[i], 1);
      mbar_init(&lnc_ready[i], 4);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 12);  // four softmax warps + eight top-G warps
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&p_full[i], 4);
      mbar_init(&o_done[i], 1);
    }
    mbar_init(fin, 1);
    mbar_init(q_ready, 4);
    *abort_s = 0;
    fence_mbar_init();
    tc::prefetch_tensormap(&maps.gK);
    tc::prefetch_tensormap(&maps.gV);
    tc::prefetch_tensormap(&maps.K);
    tc::prefetch_tensormap(&maps.V);
  }
  if (warp == 1) tc::tmem_alloc(tmem_slot, 512);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
    if (*abort_s) return false;
    if (mbar_wait(bar, parity, a.status)) return true;
    *abort_s = 1;
    return false;
  };
  const uint64_t l2pol = l2_policy_evict_first();

  if (warp < 4) regs_dec<kRegCtl>();  // (each warpgroup's branch opens with its register count)
  if (warp == 0) {
    // ================================================================ producer
    const int32_t* gM = a.gMeta + grow0;
    int kissued = 0, vissued = 0;
    for (int i = 0; i < ntile; ++i) {
      const int st = i & 1;
      unsigned char* kd = Kring + st * kTileBytes;
      unsigned char* vd = Vring + st * kTileBytes;
      const bool grp = i < gt, snk = !grp && i < gt + st_;
      const int pos = grp ? 0 : (snk ? (i - gt) * 128 : (int)(ws + (int64_t)(i - gt - st_) * 128));
      const int row = grp ? (int)(grow0 + (int64_t)i * 128) : 0;
      if (i >= 2 && !wait(&kempty[st], ((i - 2) >> 1) & 1)) break;
      if (lane == 0) {
        mbar_arrive_expect(&kfull[st], kTileBytes);
        if (grp) {
          tc::tma_load_2d(kd, &maps.gK, 0, row, &kfull[st], l2pol);
          tc::tma_load_2d(kd + kHalf, &maps.gK, 64, row, &kfull[st], l2pol);
        } else {
          tc::tma_load_4d(kd, &maps.K, 0, pos, kvh, b, &kfull[st], l2pol);
          tc::tma_load_4d(kd + kHalf, &maps.K, 64, pos, kvh, b, &kfull[st], l2pol);
        }
      }
      ++kissued;
      if (i >= 2 && !wait(&vempty[st], ((i - 2) >> 1) & 1)) break;
      if (lane == 0) {
        mbar_arrive_expect(&vfull[st], kTileBytes);
        if (grp) {
          tc::tma_load_2d(vd, &maps.gV, 0, row, &vfull[st], l2pol);
          tc::tma_load_2d(vd + kHalf, &maps.gV, 64, row, &vfull[st], l2pol);
        } else {
          tc::tma_load_4d(vd, &maps.V, 0, pos, kvh, b, &vfull[st], l2pol);
          tc::tma_load_4d(vd + kHalf, &maps.V, 64, pos, kvh, b, &vfull[st], l2pol);
        }
      }
      if (grp) {  // the groups' size and page range (zero past the visible ones)
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          const int r = lane + 32 * k4;
          const int64_t gid = (int64_t)i * 128 + r;
          const bool v = gid < G_vis;
          cp_async4_zfill(meta_s + st * 128 + r, v ? gM + gid : gM, v);
        }
      }
      cp_async_mbar_arrive_noinc(&vfull[st]);
      ++vissued;
    }
    cp_async_wait_all();
    if (*abort_s && lane == 0) {  // copies still in flight land before the CTA ends
      for (int i = kissued - 1; i >= 0 && i >= kissued - 2; --i)
        (void)mbar_wait(&kfull[i & 1], (uint32_t)(i >> 1) & 1u, a.status);
      for (int i = vissued - 1; i >= 0 && i >= vissued - 2; --i)
        (void)mbar_wait(&vfull[i & 1], (uint32_t)(i >> 1) & 1u, a.status);
    }
  } else if (warp == 1) {
    // ================================================================ MMA issue
    if (lane == 0) {
      const uint32_t idS = tc::idesc_bf16(128, 128, false, false);
      const uint32_t idO = tc::idesc_bf16(128, 128, false, true);
      const uint32_t qb = smem_u32(Qs);
      auto mma2 = [&](int j) -> bool {  // O += P_j V_j (P_j from tensor memory)
        if (!wait(&p_full[j & 1], (uint32_t)(j >> 1) & 1u)) return false;
        if (!wait(&vfull[j & 1], (uint32_t)(j >> 1) & 1u)) return false;
        tc::fence_after_sync();
        const uint32_t vb = smem_u32(Vring + (j & 1) * kTileBytes);
        const uint32_t pt = tmem + kColP + 64 * (uint32_t)(j & 1);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t bd = tc::desc_mnmajor_sw128(vb + kk * 2048, kHalf);
          tc::mma_bf16_ts(tmem + kColO, pt + 8 * kk, bd, idO, j > 0 || kk > 0);
        }
        tc::mma_commit(&vempty[j & 1]);
        tc::mma_commit(&o_done[j & 1]);
        return true;
      };
      bool go = wait(q_ready, 0), any = false;  // the query tile, staged by the softmax warps
      for (int i = 0; i < ntile && go; ++i) {
        if (!wait(&kfull[i & 1], (uint32_t)(i >> 1) & 1u)) break;
        if (i >= 2 && !wait(&s_free[i & 1], (uint32_t)((i - 2) >> 1) & 1u)) break;
        tc::fence_after_sync();
        const uint32_t kb = smem_u32(Kring + (i & 1) * kTileBytes);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t ad = tc::desc_kmajor_sw128(qb + (kk >> 2) * kHalf + (kk & 3) * 32);
          const uint64_t bd = tc::desc_kmajor_sw128(kb + (kk >> 2) * kHalf + (kk & 3) * 32);
          tc::mma_bf16(tmem + (uint32_t)(i & 1) * 128, ad, bd, idS, kk > 0);
        }
        tc::mma_commit(&kempty[i & 1]);
        tc::mma_commit(&s_full[i & 1]);
        any = true;
        if (i >= 1) go = mma2(i - 1);
        if (go && i == ntile - 1) go = mma2(i);
      }
      if (any) {
        tc::mma_commit(fin);
        (void)mbar_wait(fin, 0, a.status);
      }
    }
    __syncwarp();
  } else if (warp < 4) {
    // (warps 2 and 3: no role)
  } else if (warp < 8) {
    // ================================================================ softmax (warps 4-7)
    regs_inc<kRegSoft>();
    const int q4 = warp & 3;
    const int r = 32 * q4 + lane;  // query row of this thread (and the key row it stages)
    const uint32_t tl = (uint32_t)(32 * q4) << 16;
    {
      // the query tile, row r of MMA 1's A operand (128-byte swizzled, like
      // a key tile): row r = position r / g, head r % g
      const int64_t pi = pos0 + r / a.g;
      const int hq = kvh * a.g + r % a.g;
      const bool okr = pi < pos_end;
      const __nv_bfloat16* src = a.q + (((int64_t)b * a.Hq + hq) * a.Tq + (okr ? pi : 0)) * D;
      uint4 qw[16];
#pragma unroll
      for (int c = 0; c < 16; ++c)
        qw[c] = okr ? __ldg(reinterpret_cast<const uint4*>(src) + c) : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int c = 0; c < 16; ++c) *reinterpret_cast<uint4*>(Qs + (c >> 3) * kHalf + sw_off(r, c)) = qw[c];
      tc::fence_proxy_async();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(q_ready);
    }
    const int64_t t_row = a.q_begin + pos0 + r / a.g;
    const float scl = a.scale_log2;
    float m = -INFINITY, l = 0.f;
    bool alive = true;
    for (int i = 0; i < ntile; ++i) {
      const int st = i & 1;
      const bool grp = i < gt, snk = !grp && i < gt + st_;
      const int64_t kpos0 = grp ? 0 : (snk ? (int64_t)(i - gt) * 128 : ws + (int64_t)(i - gt - st_) * 128);
      // (a failed wait in a group tile is carried to that tile's barrier,
      // where the eight warps leave the loop together)
      alive = __all_sync(0xffffffffu, wait(&s_full[st], (uint32_t)(i >> 1) & 1u) &&
                                          wait(&vfull[st], (uint32_t)(i >> 1) & 1u));
      if (!alive && !grp) break;
      // key row r of this tile: its bias (group tiles) and whether it is in
      // no row's softmax (its value row is then zeroed: MMA 2 must not meet
      // NaN or Inf from rows that are not inputs of this call)
      bool dead = false;
      if (!alive) {
      } else if (grp) {
        const int mt = meta_s[st * 128 + r];
        const int c = mt & 0xffff;
        const int64_t gid = (int64_t)i * 128 + r;
        const bool okg = gid < G_vis && c > 0 && c <= kChunk;
        if (gid < G_vis && c > kChunk) set_status(a.status, LOD_ST_BAD_COUNT);
        lnc_s[st * 128 + r] = okg ? log2f((float)c) : -INFINITY;
        dead = !okg;
      } else {
        const int64_t kp = kpos0 + r;
        dead = snk ? kp >= nsk : kp > t_max;
      }
      if (dead) {
        unsigned char* vd = Vring + st * kTileBytes;
#pragma unroll
        for (int c = 0; c < 16; ++c)  // (swizzled order: the warp's rows spread over the banks)
          *reinterpret_cast<uint4*>(vd + (c >> 3) * kHalf + sw_off(r, c)) = make_uint4(0, 0, 0, 0);
      }
      if (grp) {  // every group's ln count is in lnc_s past here
        if (bar_red_or(kBarLncA, 128, !alive)) {
          alive = false;
          break;
        }
        if (lane == 0) mbar_arrive(&lnc_ready[st]);
      }
      tc::fence_after_sync();
      const uint32_t sb = tmem + tl + (uint32_t)st * 128;
      const float* lc = lnc_s + st * 128;
      // window and sink keys at positions kpos0 + j <= lim are in this row's softmax
      const int64_t lim = snk ? nsk - 1 : t_row;
      const int rel = grp ? 127 : (int)(lim - kpos0 < -1 ? -1 : (lim - kpos0 > 127 ? 127 : lim - kpos0));
      // the logits (log2 units) of key columns [32 c, 32 c + 32), minus `sub`
      // (one copy of the code: the loops over chunks are not unrolled)
      auto logits = [&](int c, float (&y)[32], float sub) {
        tc::tmem_ld32(sb + 32 * c, y);
        if (grp) {
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) {
            const float4 l4 = *reinterpret_cast<const float4*>(lc + 32 * c + 4 * e4);
            const float lv[4] = {l4.x - sub, l4.y - sub, l4.z - sub, l4.w - sub};
#pragma unroll
            for (int e = 0; e < 4; ++e)  // fmaxf drops NaN: a group outside the softmax gives -inf
              y[4 * e4 + e] = fmaxf(fmaf(y[4 * e4 + e], scl, lv[e]), -INFINITY);
          }
        } else {
          const int rc = rel - 32 * c;  // columns e <= rc are in
#pragma unroll
          for (int e = 0; e < 32; ++e) y[e] = e <= rc ? fmaf(y[e], scl, -sub) : -INFINITY;
        }
      };
      // Weights 2^(logit - m) into P, in one pass against the current
      // reference max m: a chunk with a logit above m + kTau2 (and a row's
      // first tile) sends the warp through the max pass first, after which
      // the weights are computed again.  Both give the same weights
      // whenever the reference max does not move.
      bool redo = __any_sync(0xffffffffu, m == -INFINITY);
      bool waited = false;
      float la[4];  // independent sum chains
      for (int att = 0; att < 2; ++att) {
        if (redo) {
          // ---- the logit max of the tile
          float xa[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};  // independent max chains
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            float y[32];
            logits(c, y, 0.f);
#pragma unroll
            for (int e = 0; e < 32; ++e) xa[e & 3] = fmaxf(xa[e & 3], y[e]);
          }
          const float xm = fmaxf(fmaxf(xa[0], xa[1]), fmaxf(xa[2], xa[3]));
          // the reference max moves when a logit exceeds it by more than kTau2
          const bool need = xm > m + kTau2;
          if (__any_sync(0xffffffffu, need)) {
            const float mn = need ? xm : m;
            const float corr = (m == -INFINITY) ? 0.f : ex2_approx(m - mn);
            l *= corr;
            m = mn;
            if (i > 0) {
              alive = __all_sync(0xffffffffu, wait(&o_done[(i - 1) & 1], (uint32_t)((i - 1) >> 1) & 1u));
              waited = true;
              if (alive) {
                tc::fence_after_sync();
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                  float ov[32];
                  tc::tmem_ld32(tmem + tl + kColO + 32 * c, ov);
#pragma unroll
                  for (int e = 0; e < 32; ++e) ov[e] *= corr;
                  tc::tmem_st32(tmem + tl + kColO + 32 * c, ov);
                }
              }
            }
          }
        }
        // P's buffer i & 1 is free once MMA 2 of tile i - 2 is done (a wait
        // for tile i - 1 above covers it)
        if (i > 1 && !waited) {
          alive = __all_sync(0xffffffffu, wait(&o_done[i & 1], (uint32_t)((i - 2) >> 1) & 1u)) && alive;
          waited = true;
        }
        if (!alive) break;
        const float mu = m == -INFINITY ? 0.f : m;
        la[0] = la[1] = la[2] = la[3] = 0.f;
        bool bail = false;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          float y[32];
          logits(c, y, mu);
          if (!redo) {  // would this chunk move the reference max?
            float ym[4] = {y[0], y[1], y[2], y[3]};
#pragma unroll
            for (int e = 4; e < 32; ++e) ym[e & 3] = fmaxf(ym[e & 3], y[e]);
            if (__any_sync(0xffffffffu, fmaxf(fmaxf(ym[0], ym[1]), fmaxf(ym[2], ym[3])) > kTau2)) {
              bail = true;
              break;
            }
          }
          uint32_t pw[16];  // the chunk's weights as bf16 pairs: columns 16 c .. 16 c + 15 of P
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float p[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              p[e] = ex2_approx(y[8 * q + e]);
              la[e & 3] += p[e];
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) pw[4 * q + e] = pack_bf16x2(p[2 * e], p[2 * e + 1]);
          }
          tmem_st16(tmem + tl + kColP + 64 * (uint32_t)st + 16 * c, pw);
        }
        if (!bail) break;
        redo = true;
      }
      if (!alive) break;
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[st]);
      l += (la[0] + la[1]) + (la[2] + la[3]);
      tmem_st_wait();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[st]);
    }
    // the row's softmax state goes to the selection warps, which write it
    ml_s[r] = alive ? make_float2(m, l) : make_float2(-INFINITY, 0.f);
    bar_named_sync(kBarEpiA, 256);
  } else {
    // ================================================================ top-G (warps 8-15) and epilogue (8-11)
    regs_inc<kRegSel>();
    const int q4 = warp & 3;
    const int r = 32 * q4 + lane;
    const int half = (warp - 8) >> 2;  // key columns [64 half, 64 half + 64) of every group tile
    const uint32_t tl = (uint32_t)(32 * q4) << 16;
    const int64_t pi = pos0 + r / a.g;
    const int hq = kvh * a.g + r % a.g;
    const bool valid = pi < pos_end;
    const float scl = a.scale_log2;
    float ts[GM];
    int ti[GM];
#pragma unroll
    for (int k = 0; k < GM; ++k) {
      ts[k] = k < GM - a.G ? INFINITY : -INFINITY;
      ti[k] = -1;
    }
    float thr = -INFINITY;
    // this row's buffer of candidates (scores above the running G-th best,
    // not yet merged into the sorted list ts/ti)
    float2* cbuf = cand_s + (half * 128 + r) * (kCandCap + 1);
    int ncand = 0;
    bool alive = true;
    for (int i = 0; i < ntile; ++i) {
      const int st = i & 1;
      const bool grp = i < gt;
      alive = __all_sync(0xffffffffu, wait(&s_full[st], (uint32_t)(i >> 1) & 1u));
      if (alive && grp) alive = __all_sync(0xffffffffu, wait(&lnc_ready[st], (uint32_t)(i >> 1) & 1u));
      if (!alive) break;
      if (grp) {
        tc::fence_after_sync();
        const float* lc = lnc_s + st * 128 + 64 * half;
#pragma unroll 1
        for (int c2 = 0; c2 < 2; ++c2) {
          float v[32];
          tc::tmem_ld32(tmem + tl + (uint32_t)st * 128 + 64 * half + 32 * c2, v);
          // the raw scores of the groups in the softmax (-inf: outside)
          float ca[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) {
            const float4 l4 = *reinterpret_cast<const float4*>(lc + 32 * c2 + 4 * e4);
            const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              float& y = v[4 * e4 + e];
              y = (valid && lv[e] != -INFINITY) ? y : -INFINITY;
              ca[e] = fmaxf(ca[e], y);
            }
          }
          const float cm = fmaxf(fmaxf(ca[0], ca[1]), fmaxf(ca[2], ca[3]));
          // candidates: scores above the running G-th best go to the buffer
          // (merged into the sorted list whenever 16 more might not fit)
          if (__any_sync(0xffffffffu, cm > thr)) {
            const int id0 = i * 128 + 64 * half + 32 * c2;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              if (__any_sync(0xffffffffu, ncand > kCandCap - 16)) topk_merge<GM>(ts, ti, thr, ncand, cbuf);
#pragma unroll
              for (int e = 16 * hh; e < 16 * hh + 16; ++e) {  // (predicated: only hits reach shared memory)
                const float y = v[e];
                const bool hit = y > thr;
                sts_f2_if(cbuf + ncand, y, __int_as_float(id0 + e), hit);
                ncand += hit ? 1 : 0;
              }
            }
          }
        }
        if (i == gt - 1) topk_merge<GM>(ts, ti, thr, ncand, cbuf);  // this half's list is final
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[st]);
    }
    // ---- the two halves' lists into one (warpgroup 3 hands its list over)
    float2* hand = cand_s + (128 + r) * (kCandCap + 1);  // (warpgroup 3's buffer, free now)
    if (half == 1) {
#pragma unroll
      for (int k = 0; k < GM; ++k) hand[k] = make_float2(ts[k], __int_as_float(ti[k]));
      hand[GM] = make_float2(alive ? 1.f : 0.f, 0.f);
    }
    bar_named_sync(kBarSelA, 256);
    if (half == 1) return;  // (warpgroup 3 is done; the CTA's last barrier counts warpgroups 0-2 only)
    if (hand[GM].x == 0.f) alive = false;
#pragma unroll
    for (int k = 0; k < GM; ++k) {
      const float2 e = hand[k];
      const int id = __float_as_int(e.y);
      if (id >= 0) topk_insert_ranked<GM>(ts, ti, e.x, id);
    }
    // ---------------------------------------------------------------- epilogue
    bar_named_sync(kBarEpiA, 256);
    const float2 ml = ml_s[r];
    const float m = ml.x;
    float l = ml.y;
    if (ml.x == -INFINITY && ml.y == 0.f && gt + st_ < ntile) alive = false;  // the softmax gave up
    if (alive && ntile > 0)
      alive = __all_sync(0xffffffffu, wait(&o_done[(ntile - 1) & 1], (uint32_t)((ntile - 1) >> 1) & 1u));
    tc::fence_after_sync();
    const int64_t wr = ((int64_t)b * a.Hq + hq) * a.NW + (pi - a.w_lo);  // wave row
    const int64_t orow = ((int64_t)b * a.Hq + hq) * a.Tq + pi;
    // the row state (m, l, acc) and the opened groups (list slots GM - G ..
    // GM - 1, best first, -1: none) with the weights of their coarse terms
    // relative to m: the merge removes those terms (finer entries replace them)
    float* stp = a.state + wr * kStateStride;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float ov[32];
      tc::tmem_ld32(tmem + tl + kColO + 32 * c, ov);
      if (valid && alive) {
#pragma unroll
        for (int q = 0; q < 8; ++q)
          *reinterpret_cast<float4*>(stp + 4 + 32 * c + 4 * q) =
              make_float4(ov[4 * q], ov[4 * q + 1], ov[4 * q + 2], ov[4 * q + 3]);
      }
    }
    if (valid) {
      // the pairs' places in their groups' runs: every atomic is issued
      // before any result is used, so their round trips overlap
      int pos[GM];
#pragma unroll
      for (int k = 0; k < GM; ++k) {
        const int gid = alive ? ti[k] : -1;
        pos[k] = (k >= GM - a.G && gid >= 0) ? atomicAdd(a.cnt + grow0 + gid, 1) : -1;
      }
      // the groups' sizes, all loads in flight together (the stores below
      // would otherwise keep each load behind the previous one's stores)
      int gsz[GM];
#pragma unroll
      for (int k = 0; k < GM; ++k) {
        const int gid = alive ? ti[k] : -1;
        gsz[k] = (k >= GM - a.G && gid >= 0) ? __ldg(a.gMeta + grow0 + gid) & 0xffff : 0;
      }
      *reinterpret_cast<float2*>(stp) = alive ? make_float2(m, l) : make_float2(-INFINITY, 0.f);
      const float mu = m == -INFINITY ? 0.f : m;
#pragma unroll
      for (int k = 0; k < GM; ++k) {
        if (k >= GM - a.G) {
          const int j = k - (GM - a.G);  // rank
          const int gid = alive ? ti[k] : -1;
          float wk = 0.f;
          if (gid >= 0) {
            const int c = gsz[k];
            wk = ex2_approx(fmaf(ts[k], scl, log2f((float)(c > 0 ? c : 1))) - mu);
          }
          a.sel[wr * a.G + j] = gid;
          a.cw[wr * a.G + j] = wk;
          a.pos[wr * a.G + j] = pos[k];
          if (a.sel_groups) a.sel_groups[orow * a.G + j] = gid;
        }
      }
    }
  }
  tc::fence_before_sync();
  bar_named_sync(kBarEndA, 384);  // warpgroups 0-2 (warpgroup 3 has left)
  if (warp == 1) tc::tmem_dealloc(tmem, 512);
}

// ================================================================== plan, scatter

constexpr int kPlanThreads = 1024;

// Exclusive prefix sums of the per-group pair counts (off) and the work
// items: group gflat with c pairs gives ceil(c / item_rows) items
// {gflat, first pair, pairs}.
__global__ void __launch_bounds__(kPlanThreads) pf_plan_kernel(const __grid_constant__ PrefillArgs a) {
  __shared__ int wsum[3][32];
  __shared__ long long carry[3];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid < 3) carry[tid] = 0;
  __syncthreads();
  for (int64_t base = 0; base < a.Gtot; base += kPlanThreads) {
    const int64_t gf = base + tid;
    const int c = gf < a.Gtot ? a.cnt[gf] : 0;
    const bool big = c > 0 && (a.gMeta[gf] & 0xffff) > kSmallN;
    const int ni = (c + a.item_rows - 1) / a.item_rows;
    int x[3] = {c, big ? 0 : ni, big ? ni : 0};  // pairs, small items, big items
    int y[3] = {x[0], x[1], x[2]};                // inclusive warp scans
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
      for (int q = 0; q < 3; ++q) {
        const int z = __shfl_up_sync(0xffffffffu, y[q], o);
        if (lane >= o) y[q] += z;
      }
    }
    if (lane == 31) {
#pragma unroll
      for (int q = 0; q < 3; ++q) wsum[q][warp] = y[q];
    }
    __syncthreads();
    if (warp == 0) {
#pragma unroll
      for (int q = 0; q < 3; ++q) {
        int sv = wsum[q][lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int z = __shfl_up_sync(0xffffffffu, sv, o);
          if (lane >= o) sv += z;
        }
        wsum[q][lane] = sv;
      }
    }
    __syncthreads();
    long long ex[3];
#pragma unroll
    for (int q = 0; q < 3; ++q) ex[q] = carry[q] + (warp > 0 ? wsum[q][warp - 1] : 0) + y[q] - x[q];
    if (gf < a.Gtot) {
      a.off[gf] = (int32_t)ex[0];
      int4* dst = big ? a.items + a.big_items + ex[2] : a.items + ex[1];
      for (int t = 0; t < ni; ++t) {
        const int n = c - t * a.item_rows < a.item_rows ? c - t * a.item_rows : a.item_rows;
        dst[t] = make_int4((int)gf, (int)(ex[0] + (long long)t * a.item_rows), n, 0);
      }
    }
    __syncthreads();
    if (tid < 3) carry[tid] += wsum[tid][31];
    __syncthreads();
  }
  if (tid == 0) {
    a.n_items[0] = (int32_t)carry[1];
    a.n_items[1] = (int32_t)carry[2];
  }
}

// Every (row, group) pair into its group's run of the pair list, at the
// place its counting atomic returned (the order inside a run is arbitrary:
// every pair is computed on its own).
__global__ void __launch_bounds__(256) pf_scatter_kernel(const __grid_constant__ PrefillArgs a) {
  // (32-bit index arithmetic: the wave's pairs number fewer than 2^31)
  const int n = a.B * a.Hq * (int)a.NW * a.G;
  const int NW = (int)a.NW;
  for (int idx = blockIdx.x * 256 + threadIdx.x; idx < n; idx += gridDim.x * 256) {
    const int gid = a.sel[idx];
    if (gid < 0) continue;
    const int wr = idx / a.G;
    const int bh = wr / NW;
    const int pr = wr - bh * NW;
    if (a.w_lo + pr >= a.w_hi) continue;
    const int64_t u = (int64_t)(bh / a.Hq) * a.Hkv + (bh % a.Hq) / a.g;
    const int64_t at = a.off[u * a.Cmax * a.k + gid] + a.pos[idx];
    a.list[at] = (int32_t)idx;
    a.list_q[at] = (int32_t)(bh * a.Tq + a.w_lo + pr);  // the pair's row of q / out
  }
}

// ================================================================== phase B

constexpr int kThreadsB = 160;   // warp 0 TMA + MMA issue, warps 1-4 one pair per thread
constexpr int kBarSoftB = 2;

// Shared memory and tensor memory of the pair kernel.  SMALL (groups of at
// most kSmallN members, two CTAs per SM): a fixed 104 KB layout, the query
// tile and P share one region (P is written after S has been computed), S
// in TMEM columns [0, 128), O in [128, 256) with the page scores in its
// first 16 columns until MMA 2 overwrites them.  BIG (one CTA per SM, up to
// a whole chunk): the layout follows the group size, S in [0, 256), the
// page scores in [256, 272), O in [384, 512).
template <bool BIG>
struct PairCfg {
  static constexpr size_t kData = BIG ? 216 * 1024 : 104 * 1024;
  static constexpr uint32_t kTmemCols = BIG ? 512 : 256;
  static constexpr uint32_t kColSp = BIG ? 256 : 128;
  static constexpr uint32_t kColO = BIG ? 384 : 128;
  static constexpr size_t off_misc = kData;            // per-item info
  static constexpr size_t off_lpc = off_misc + 96;     // float [16] log2 page counts
  static constexpr size_t off_bar = off_lpc + 64;
  static constexpr int kBars = 6;
  static constexpr size_t off_tmem = off_bar + 8 * kBars;
  static constexpr size_t bytes = off_tmem + 16 + 1024;
  static_assert(bytes <= (BIG ? 227 * 1024 : 113 * 1024), "shared memory of the CTAs of one SM");
};

struct ItemInfo {
  int n, np, p0, ok;
  int start, count, R, shared_qp;
  int64_t c, u;
  uint32_t off_kg, off_vg, off_q, off_p;
};

template <bool BIG>
__global__ void __launch_bounds__(kThreadsB, BIG ? 1 : 2)
    pf_pair_kernel(const __grid_constant__ PairMaps maps, const __grid_constant__ PrefillArgs a) {
  using Cfg = PairCfg<BIG>;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                       ~uintptr_t(1023));
  ItemInfo* info = reinterpret_cast<ItemInfo*>(sm + Cfg::off_misc);
  float* lpc_s = reinterpret_cast<float*>(sm + Cfg::off_lpc);
  uint64_t* gfull = reinterpret_cast<uint64_t*>(sm + Cfg::off_bar);
  uint64_t* q_full = gfull + 1;
  uint64_t* s_full = q_full + 1;
  uint64_t* p_full = s_full + 1;
  uint64_t* o_done = p_full + 1;
  uint64_t* o_free = o_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + Cfg::off_tmem);
  unsigned char* PKs = sm;             // [2 halves][16 rows][128 B]
  unsigned char* PVs = sm + 4096;

  if (tid == 0) {
    mbar_init(gfull, 1);
    mbar_init(q_full, 128);
    mbar_init(s_full, 1);
    mbar_init(p_full, 4);
    mbar_init(o_done, 1);
    mbar_init(o_free, 4);
    fence_mbar_init();
    tc::prefetch_tensormap(&maps.mK);
    tc::prefetch_tensormap(&maps.mV);
    tc::prefetch_tensormap(&maps.pK);
    tc::prefetch_tensormap(&maps.pV);
  }
  if (warp == 0) tc::tmem_alloc(tmem_slot, Cfg::kTmemCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const int n_items = a.n_items[BIG ? 1 : 0];
  const int4* items = a.items + (BIG ? a.big_items : 0);
  const int64_t Gcap = a.Cmax * a.k;
  const float scl = a.scale_log2;
  const int G = a.G, TP = a.TP;
  uint32_t T = 0;      // tiles processed by this CTA (barrier phases)
  uint32_t ngrp = 0;   // items processed (gfull phases)
  bool alive = true;
  // (thread 0 reads each item and its group word one item ahead)
  int4 nx_item = make_int4(0, 0, 0, 0);
  int nx_meta = 0;
  if (tid == 0 && (int)blockIdx.x < n_items) {
    nx_item = items[blockIdx.x];
    nx_meta = a.gMeta[nx_item.x];
  }

  for (int it = blockIdx.x; it < n_items && alive; it += gridDim.x) {
    // ---- the item: its group, bounds-checked, and the operand layout
    if (tid == 0) {
      const int4 item = nx_item;
      const int meta = nx_meta;
      if (it + (int)gridDim.x < n_items) {
        nx_item = items[it + gridDim.x];
        nx_meta = a.gMeta[nx_item.x];
      }
      const int64_t gflat = item.x;
      const int64_t u = gflat / Gcap, gid = gflat % Gcap, c = gid / a.k;
      const int n = meta & 0xffff, p0 = (meta >> 16) & 0xff, p1 = (meta >> 24) & 0xff;
      const int64_t pslot = (u * a.Cmax + c) * a.P;
      bool ok = n >= 1 && n <= (BIG ? kChunk : kSmallN) && p0 < p1 && p1 <= a.P && p1 - p0 == (n + kPage - 1) / kPage;
      if (!ok) set_status(a.status, n > kChunk ? LOD_ST_BAD_COUNT : LOD_ST_BAD_PAGE);
      const int off = ok ? (int)a.pBeg[pslot + p0] : 0;
      if (ok && (off < 0 || off + n > kChunk)) {
        set_status(a.status, LOD_ST_BAD_MEMBER);
        ok = false;
      }
      ItemInfo f;
      f.n = ok ? n : 16;
      f.np = ok ? p1 - p0 : 1;
      f.p0 = p0;
      f.ok = ok;
      f.start = item.y;
      f.count = item.z;
      f.c = c;
      f.u = u;
      f.R = ok ? (n + 31) / 32 * 32 : 32;
      const uint32_t kg = BIG ? (uint32_t)f.R * 256 : 128 * 256;  // one operand: 2 halves x R rows x 128 B
      const int n16 = (f.n + 15) / 16 * 16;
      const uint32_t pbytes = (uint32_t)((n16 + 16 + 63) / 64) * kHalf;
      f.off_kg = 8192;
      f.off_vg = 8192 + kg;
      f.off_q = 8192 + 2 * kg;
      f.shared_qp = !BIG || f.off_q + kTileBytes + pbytes > Cfg::kData;
      f.off_p = f.shared_qp ? f.off_q : f.off_q + kTileBytes;
      *info = f;
      const int rs = BIG ? f.R : 128;  // rows of one operand half in shared memory
      if (ok) {
        mbar_arrive_expect(gfull, 2 * (uint32_t)f.R * 256 + 2 * 4096);
        const int row0 = (int)((u * a.Cmax + c) * kChunk + off);
        for (int bx = 0; bx < f.R / 32; ++bx)
          for (int h = 0; h < 2; ++h) {
            tc::tma_load_2d(sm + f.off_kg + h * (rs * 128) + bx * 4096, &maps.mK, 64 * h, row0 + 32 * bx, gfull,
                            0x1000000000000000ull);
            tc::tma_load_2d(sm + f.off_vg + h * (rs * 128) + bx * 4096, &maps.mV, 64 * h, row0 + 32 * bx, gfull,
                            0x1000000000000000ull);
          }
        for (int h = 0; h < 2; ++h) {
          tc::tma_load_2d(PKs + h * 2048, &maps.pK, 64 * h, (int)(pslot + p0), gfull, 0x1000000000000000ull);
          tc::tma_load_2d(PVs + h * 2048, &maps.pV, 64 * h, (int)(pslot + p0), gfull, 0x1000000000000000ull);
        }
      } else {
        mbar_arrive(gfull);
      }
    }
    __syncthreads();
    const ItemInfo f = *info;
    const int n16 = (f.n + 15) / 16 * 16;
    const int ntiles = (f.count + kRows - 1) / kRows;
    const int rs = BIG ? f.R : 128;
    unsigned char* KG = sm + f.off_kg;
    unsigned char* VG = sm + f.off_vg;
    unsigned char* Qs = sm + f.off_q;
    unsigned char* Ps = sm + f.off_p;

    if (warp == 0) {
      // ============================================================ MMA issue
      if (lane == 0) {
        bool go = mbar_wait(gfull, ngrp & 1u, a.status);
        const uint32_t idS = tc::idesc_bf16(128, n16, false, false);
        const uint32_t idP = tc::idesc_bf16(128, 16, false, false);
        const uint32_t idO = tc::idesc_bf16(128, 128, false, true);
        const uint32_t qb = smem_u32(Qs), kb = smem_u32(KG), vb = smem_u32(VG), pb = smem_u32(Ps);
        const uint32_t pkb = smem_u32(PKs), pvb = smem_u32(PVs);
        const uint32_t hs = (uint32_t)rs * 128;
        for (int t = 0; t < ntiles && go; ++t) {
          const uint32_t Tt = T + t;
          go = mbar_wait(q_full, Tt & 1u, a.status);
          // (O is free once the epilogue of the previous tile has read it; the
          // page scores share its columns in the SMALL layout)
          if (go && Tt > 0) go = mbar_wait(o_free, (Tt - 1) & 1u, a.status);
          if (!go) break;
          tc::fence_after_sync();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t ad = tc::desc_kmajor_sw128(qb + (kk >> 2) * kHalf + (kk & 3) * 32);
            tc::mma_bf16(tmem, ad, tc::desc_kmajor_sw128(kb + (kk >> 2) * hs + (kk & 3) * 32), idS, kk > 0);
            tc::mma_bf16(tmem + Cfg::kColSp, ad, tc::desc_kmajor_sw128(pkb + (kk >> 2) * 2048 + (kk & 3) * 32), idP,
                         kk > 0);
          }
          tc::mma_commit(s_full);
          go = mbar_wait(p_full, Tt & 1u, a.status);
          if (!go) break;
          tc::fence_after_sync();
          for (int kk = 0; kk < n16 / 16; ++kk)
            tc::mma_bf16(tmem + Cfg::kColO, tc::desc_kmajor_sw128(pb + (kk >> 2) * kHalf + (kk & 3) * 32),
                         tc::desc_mnmajor_sw128(vb + kk * 2048, hs), idO, kk > 0);
          {
            const int kk = n16 / 16;  // the coarse pages' weights and mean values
            tc::mma_bf16(tmem + Cfg::kColO, tc::desc_kmajor_sw128(pb + (kk >> 2) * kHalf + (kk & 3) * 32),
                         tc::desc_mnmajor_sw128(pvb, 2048), idO, true);
          }
          tc::mma_commit(o_done);
        }
        if (!go) set_status(a.status, LOD_ST_TIMEOUT);
      }
      __syncwarp();
    } else {
      // ============================================================ pairs
      const int q4 = warp & 3;
      const int r = 32 * q4 + lane;
      const uint32_t tl = (uint32_t)(32 * q4) << 16;
      // the query row of pair t * 128 + r, staged by this thread
      // the pair list entries of tile t (read one tile ahead of its gather)
      auto entries = [&](int t, int& pid, int& qrow) {
        const int idx = t * kRows + r;
        const bool v = idx < f.count;
        pid = v ? a.list[f.start + idx] : -1;
        qrow = v ? a.list_q[f.start + idx] : 0;
      };
      auto gather = [&](int t, int pid, int qrow) {
        const bool v = pid >= 0;
        const __nv_bfloat16* src = a.q + (int64_t)qrow * D;
#pragma unroll
        for (int c = 0; c < 16; ++c)
          cp_async16_zfill(Qs + (c >> 3) * kHalf + sw_off(r, c), reinterpret_cast<const uint4*>(src) + c, v);
        cp_async_mbar_arrive_noinc(q_full);
      };
      int pid_cur = -1, pid_next = -1, qr_cur = 0, qr_next = 0;
      entries(0, pid_cur, qr_cur);
      gather(0, pid_cur, qr_cur);
      // page counts of the group (log2, for the coarse logits)
      if (r < 16) {
        float v = -INFINITY;
        if (f.ok && r < f.np) {
          const int pc = a.pCnt[(f.u * a.Cmax + f.c) * a.P + f.p0 + r];
          if (pc > 0 && pc <= kPage) v = log2f((float)pc);
          else set_status(a.status, LOD_ST_BAD_COUNT);
        }
        lpc_s[r] = v;
      }
      // rows past the group's members, and page slots past its pages, are
      // not inputs of this group: zero their values for MMA 2
      alive = mbar_wait(gfull, ngrp & 1u, a.status);
      if (alive) {
        const int hs = rs * 128;
        for (int x = r; x < (n16 - f.n) * 16; x += 128) {
          const int row = f.n + x / 16, ch = x % 16;
          *reinterpret_cast<uint4*>(VG + (ch >> 3) * hs + sw_off(row, ch)) = make_uint4(0, 0, 0, 0);
        }
        for (int x = r; x < (16 - f.np) * 16; x += 128) {
          const int row = f.np + x / 16, ch = x % 16;
          *reinterpret_cast<uint4*>(PVs + (ch >> 3) * 2048 + sw_off(row, ch)) = make_uint4(0, 0, 0, 0);
        }
        tc::fence_proxy_async();
      }
      bar_named_sync(kBarSoftB, 128);
      const int nblk = (f.np + 3) / 4;  // 64-column blocks of member scores (4 pages each)
      for (int t = 0; t < ntiles && alive; ++t) {
        const uint32_t Tt = T + t;
        alive = __all_sync(0xffffffffu, mbar_wait(s_full, Tt & 1u, a.status));
        if (!alive) break;
        tc::fence_after_sync();
        if (t + 1 < ntiles) entries(t + 1, pid_next, qr_next);
        if (t + 1 < ntiles && !f.shared_qp) gather(t + 1, pid_next, qr_next);
        // page scores and this row's top-TP pages (score desc, slot asc)
        float sp[16];
        tc::tmem_ld16(tmem + tl + Cfg::kColSp, sp);
        uint32_t selm = 0;
        if (TP == 0 || TP >= f.np) {
          selm = (1u << f.np) - 1u;
        } else {
#pragma unroll
          for (int x = 0; x < kMaxTopPages; ++x) {
            if (x < TP) {
              float bs = -INFINITY;
              int bj = -1;
#pragma unroll
              for (int j = 0; j < 16; ++j)
                if (j < f.np && !((selm >> j) & 1u) && (bj < 0 || sp[j] > bs)) {
                  bs = sp[j];
                  bj = j;
                }
              selm |= 1u << bj;
            }
          }
        }
        // pass 1: the row's max over its exact members and coarse pages
        float xc[16];
        float ma[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const bool coarse = TP > 0 && j < f.np && !((selm >> j) & 1u);
          xc[j] = coarse ? fmaf(sp[j], scl, lpc_s[j]) : -INFINITY;
          ma[j & 3] = fmaxf(ma[j & 3], xc[j]);
        }
        for (int bb = 0; bb < nblk; ++bb) {
          float v[64];
          tc::tmem_ld32xN<2>(tmem + tl + 64 * bb, v);
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            const int j = 4 * bb + jj;
            if ((selm >> j) & 1u) {
#pragma unroll
              for (int e = 0; e < 16; ++e)
                if (16 * j + e < f.n) ma[e & 3] = fmaxf(ma[e & 3], v[16 * jj + e] * scl);
            }
          }
        }
        const float m = fmaxf(fmaxf(ma[0], ma[1]), fmaxf(ma[2], ma[3]));
        const float mu = m == -INFINITY ? 0.f : m;
        // pass 2: the weights into P (members, then the coarse pages)
        float la[4] = {0.f, 0.f, 0.f, 0.f};
        for (int bb = 0; bb < nblk; ++bb) {
          float v[64];
          tc::tmem_ld32xN<2>(tmem + tl + 64 * bb, v);
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            const int j = 4 * bb + jj;
            if (j < f.np) {
              const bool on = (selm >> j) & 1u;
              float p[16];
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                p[e] = (on && 16 * j + e < f.n) ? ex2_approx(fmaf(v[16 * jj + e], scl, -mu)) : 0.f;
                la[e & 3] += p[e];
              }
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const int ch = 2 * j + h;
                *reinterpret_cast<uint4*>(Ps + (ch >> 3) * kHalf + sw_off(r, ch)) =
                    make_uint4(pack_bf16x2(p[8 * h], p[8 * h + 1]), pack_bf16x2(p[8 * h + 2], p[8 * h + 3]),
                               pack_bf16x2(p[8 * h + 4], p[8 * h + 5]), pack_bf16x2(p[8 * h + 6], p[8 * h + 7]));
              }
            }
          }
        }
        {
          float p[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            p[e] = xc[e] == -INFINITY ? 0.f : ex2_approx(xc[e] - mu);
            la[e & 3] += p[e];
          }
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int ch = n16 / 8 + h;
            *reinterpret_cast<uint4*>(Ps + (ch >> 3) * kHalf + sw_off(r, ch)) =
                make_uint4(pack_bf16x2(p[8 * h], p[8 * h + 1]), pack_bf16x2(p[8 * h + 2], p[8 * h + 3]),
                           pack_bf16x2(p[8 * h + 4], p[8 * h + 5]), pack_bf16x2(p[8 * h + 6], p[8 * h + 7]));
          }
        }
        const float l = (la[0] + la[1]) + (la[2] + la[3]);
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);
        // ---- epilogue: the pair's normalised partial
        alive = __all_sync(0xffffffffu, mbar_wait(o_done, Tt & 1u, a.status));
        if (!alive) break;
        tc::fence_after_sync();
        const bool vp = pid_cur >= 0 && f.ok;
        const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          float ov[64];
          tc::tmem_ld32xN<2>(tmem + tl + Cfg::kColO + 64 * hh, ov);
          if (hh == 1) {
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(o_free);
          }
          if (vp) {
            uint4* dst = reinterpret_cast<uint4*>(a.po + (int64_t)pid_cur * D + 64 * hh);
#pragma unroll
            for (int q = 0; q < 8; ++q)
              dst[q] = make_uint4(pack_bf16x2(ov[8 * q] * inv, ov[8 * q + 1] * inv),
                                  pack_bf16x2(ov[8 * q + 2] * inv, ov[8 * q + 3] * inv),
                                  pack_bf16x2(ov[8 * q + 4] * inv, ov[8 * q + 5] * inv),
                                  pack_bf16x2(ov[8 * q + 6] * inv, ov[8 * q + 7] * inv));
          }
        }
        if (t + 1 < ntiles && f.shared_qp) gather(t + 1, pid_next, qr_next);
        if (pid_cur >= 0) {
          a.plse[pid_cur] = vp && l > 0.f ? m + log2f(l) : -INFINITY;
          if (a.sel_pages) {
            const int rank = pid_cur - (pid_cur / G) * G;
            int32_t* spo = a.sel_pages + ((int64_t)qr_cur * G + rank) * TP;
            // the opened pages, best first (score desc, slot asc)
            uint32_t rest = vp ? selm : 0u;
            for (int x = 0; x < TP; ++x) {
              int bj = -1;
              float bs = -INFINITY;
#pragma unroll
              for (int j = 0; j < 16; ++j)
                if (((rest >> j) & 1u) && (bj < 0 || sp[j] > bs)) {
                  bs = sp[j];
                  bj = j;
                }
              spo[x] = bj >= 0 ? (int32_t)(f.c * a.P + f.p0 + bj) : -1;
              if (bj >= 0) rest &= ~(1u << bj);
            }
          }
        }
        pid_cur = pid_next;
        qr_cur = qr_next;
      }
      // (a gathered tile that was never consumed: let its copies land)
      cp_async_wait_all();
    }
    T += (uint32_t)ntiles;
    ++ngrp;
    alive = !__syncthreads_or(!alive);
  }
  if (!alive && tid == 0) set_status(a.status, LOD_ST_TIMEOUT);
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, Cfg::kTmemCols);
}

// ================================================================== merge

// One warp per row: the row state (m, l, acc), minus the opened groups'
// coarse terms, and the partials of those groups in one softmax.  Lane k
// reads rank k's bookkeeping; every value slice is requested before any is
// used, so the row's loads are in flight together.
template <int GM>
__global__ void __launch_bounds__(256) pf_merge_kernel(const __grid_constant__ PrefillArgs a) {
  const int lane = threadIdx.x & 31;
  // (32-bit index arithmetic: the wave's rows number fewer than 2^31)
  const int NW = (int)a.NW;
  const int nrows = a.B * a.Hq * NW;
  const int wr = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (wr >= nrows) return;
  const int bh = wr / NW;
  const int64_t pi = a.w_lo + (wr - bh * NW);
  if (pi >= a.w_hi) return;
  const int64_t orow = (int64_t)bh * a.Tq + pi;
  const int64_t u = (int64_t)(bh / a.Hq) * a.Hkv + (bh % a.Hq) / a.g;
  const float* stp = a.state + (int64_t)wr * kStateStride;
  const int G = a.G;
  // rank `lane`: group, coarse weight, partial's log-sum-exp
  const int gid_l = lane < G ? a.sel[wr * G + lane] : -1;
  const float cw_l = lane < G ? a.cw[wr * G + lane] : 0.f;
  const float pl_l = lane < G ? a.plse[wr * G + lane] : -INFINITY;
  const float2 ml = *reinterpret_cast<const float2*>(stp);
  const float m = ml.x;
  const float4 acc = m == -INFINITY ? make_float4(0.f, 0.f, 0.f, 0.f)
                                    : *reinterpret_cast<const float4*>(stp + 4 + 4 * lane);
  uint2 gv[GM], po[GM];
#pragma unroll
  for (int k = 0; k < GM; ++k) {
    const int gid = __shfl_sync(0xffffffffu, gid_l, k);
    gv[k] = make_uint2(0u, 0u);
    po[k] = make_uint2(0u, 0u);
    if (k < G && gid >= 0) {
      gv[k] = *reinterpret_cast<const uint2*>(a.gV + ((u * a.Cmax * a.k + gid) * D + 4 * lane));
      po[k] = *reinterpret_cast<const uint2*>(a.po + (int64_t)(wr * G + k) * D + 4 * lane);
    }
  }
  // the common max over the state and the partials
  float M = m;
  {
    const float pv = gid_l >= 0 ? pl_l : -INFINITY;
    M = fmaxf(M, warp_max(pv));
  }
  const float cs = m == -INFINITY ? 0.f : ex2_approx(m - M);
  float L = ml.y, o0 = acc.x, o1 = acc.y, o2 = acc.z, o3 = acc.w;
#pragma unroll
  for (int k = 0; k < GM; ++k) {  // the opened groups' coarse terms leave the state
    const int gid = __shfl_sync(0xffffffffu, gid_l, k);
    const float wk = __shfl_sync(0xffffffffu, cw_l, k);
    if (k < G && gid >= 0 && m != -INFINITY) {
      L -= wk;
      o0 = fmaf(-wk, __uint_as_float(gv[k].x << 16), o0);
      o1 = fmaf(-wk, __uint_as_float(gv[k].x & 0xffff0000u), o1);
      o2 = fmaf(-wk, __uint_as_float(gv[k].y << 16), o2);
      o3 = fmaf(-wk, __uint_as_float(gv[k].y & 0xffff0000u), o3);
    }
  }
  L *= cs;
  o0 *= cs;
  o1 *= cs;
  o2 *= cs;
  o3 *= cs;
#pragma unroll
  for (int k = 0; k < GM; ++k) {  // the finer entries: the pairs' partials
    const int gid = __shfl_sync(0xffffffffu, gid_l, k);
    const float ls = __shfl_sync(0xffffffffu, pl_l, k);
    if (k < G && gid >= 0 && ls != -INFINITY) {
      const float w = ex2_approx(ls - M);
      L += w;
      o0 = fmaf(w, __uint_as_float(po[k].x << 16), o0);
      o1 = fmaf(w, __uint_as_float(po[k].x & 0xffff0000u), o1);
      o2 = fmaf(w, __uint_as_float(po[k].y << 16), o2);
      o3 = fmaf(w, __uint_as_float(po[k].y & 0xffff0000u), o3);
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  *reinterpret_cast<uint2*>(a.out + orow * D + 4 * lane) =
      make_uint2(pack_bf16x2(o0 * inv, o1 * inv), pack_bf16x2(o2 * inv, o3 * inv));
  if (lane == 0 && a.lse) a.lse[orow] = (M + log2f(L)) * 0.69314718055994531f;
  // sel_pages of the ranks with no opened group (the pair kernel writes the others)
  if (a.sel_pages)
    for (int k = 0; k < G; ++k)
      if (__shfl_sync(0xffffffffu, gid_l, k) < 0 && lane < a.TP) a.sel_pages[(orow * G + k) * a.TP + lane] = -1;
}

}  // namespace

size_t prefill_tc_scan_smem() { return SmemA::bytes; }
size_t prefill_tc_pair_smem() { return PairCfg<true>::bytes; }

cudaError_t launch_prefill_tc_wave(const PrefillArgs& a, const TcMaps& maps, const PairMaps& pmaps, int num_sms,
                                   cudaStream_t stream) {
  cudaError_t e = cudaMemsetAsync(a.cnt, 0, sizeof(int32_t) * (size_t)a.Gtot, stream);
  if (e != cudaSuccess) return e;
  const int RP = kRows / a.g;
  const int64_t nblk = (a.w_hi - a.w_lo + RP - 1) / RP;
  const int64_t tiles = nblk * a.B * a.Hkv;
  if (a.G <= 8) {
    e = set_smem_once<pf_scan_kernel<8>>(SmemA::bytes);
    if (e == cudaSuccess)
      pf_scan_kernel<8><<<(unsigned)tiles, kThreadsA, SmemA::bytes, stream>>>(maps, a);
  } else {
    e = set_smem_once<pf_scan_kernel<16>>(SmemA::bytes);
    if (e == cudaSuccess)
      pf_scan_kernel<16><<<(unsigned)tiles, kThreadsA, SmemA::bytes, stream>>>(maps, a);
  }
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  pf_plan_kernel<<<1, kPlanThreads, 0, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t npairs = (int64_t)a.B * a.Hq * a.NW * a.G;
  const int64_t sblocks = (npairs + 255) / 256 < 64 * num_sms ? (npairs + 255) / 256 : 64 * num_sms;
  pf_scatter_kernel<<<(unsigned)(sblocks > 0 ? sblocks : 1), 256, 0, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = set_smem_once<pf_pair_kernel<false>>(PairCfg<false>::bytes, true);
  if (e == cudaSuccess) e = set_smem_once<pf_pair_kernel<true>>(PairCfg<true>::bytes, true);
  if (e != cudaSuccess) return e;
  pf_pair_kernel<false><<<(unsigned)(2 * num_sms), kThreadsB, PairCfg<false>::bytes, stream>>>(pmaps, a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  pf_pair_kernel<true><<<(unsigned)num_sms, kThreadsB, PairCfg<true>::bytes, stream>>>(pmaps, a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t rows = (int64_t)a.B * a.Hq * a.NW;
  if (a.G <= 8)
    pf_merge_kernel<8><<<(unsigned)((rows + 7) / 8), 256, 0, stream>>>(a);
  else
    pf_merge_kernel<16><<<(unsigned)((rows + 7) / 8), 256, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace lod
