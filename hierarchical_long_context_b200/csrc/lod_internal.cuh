// lod_internal.cuh -- argument blocks and launchers shared by the library's
// translation units (not part of the public ABI).
#pragma once

#include <cuda.h>

#include <atomic>
#include <utility>

#include "lod_common.cuh"

namespace lod {

struct BuildArgs {
  const void* K;
  const void* V;
  int64_t sb, sh, st;  // KV strides in elements (sequence, head, token)
  int Hkv;
  int64_t Cmax;        // index capacity in chunks
  int k;               // clusters
  int iters;           // Lloyd rounds
  int sinks;
  int head_shard;      // 0, or (model KV heads << 16) | this shard's first KV head
  int P;               // page slots per chunk
  int64_t chunk_begin;
  const int64_t* seq_lens;  // non-null: per sequence, the chunk its length just completed (else nothing)
  uint64_t seed;
  void* gK;
  void* gV;
  int32_t* gCnt;
  void* pK;
  void* pV;
  int32_t* pCnt;
  int16_t* pBeg;
  int16_t* gPage;
  int16_t* perm;
  void* mK;            // member-ordered key / value copies
  void* mV;
  int32_t* gMeta;      // size | first page << 16 | end page << 24 per group
  int kv_bits;         // 4: three-tier INT4 (qK/qV codes + qKs/qVs quantisers instead of mK/mV)
  uint8_t* qK;         // [..][Cmax * chunk][d / 2] member-ordered 4-bit codes
  uint8_t* qV;
  float2* qKs;         // [..][Cmax * P][d] (scale, low) per page slot and channel
  float2* qVs;
  uint32_t* status;    // device status word (workspace header)
};

// Opt kernel `Kern` in to `smem` bytes of dynamic shared memory, once per
// device (later calls make no CUDA call, so launches stay capturable in a
// graph).  The flag is per kernel: Kern is a template argument.  max_shared:
// also prefer the largest shared-memory carveout (for a kernel whose
// occupancy is set by its shared memory).
template <auto Kern>
cudaError_t set_smem_once(size_t smem, bool max_shared = false) {
  static std::atomic<uint64_t> done{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev < 64 ? (uint64_t)1 << dev : 0;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(Kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess && max_shared)
    e = cudaFuncSetAttribute(Kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_release);
  return e;
}

// Launch `kern` as a programmatic dependent of the preceding work in `stream`
// (it may start before that work completes and must call pdl_wait before
// reading anything it produced).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
  return e == cudaSuccess ? cudaGetLastError() : e;
}

// Scan CTAs a decode call aims for: two resident CTAs on each of the B200's 148 SMs.
constexpr int kTargetCtas = 2 * 148;
// Rows of one scan pipeline stage (a split streams whole stages).
constexpr int kScanSlab = 64;

// One of a scan split's best groups for one query row (tensor-core scan).
struct SplitCand {
  float s;    // scale * q . mean k
  int id;     // group id within the unit (chunk * k + slot); -1: none
  int meta;   // the group's gMeta word
  int pad;
};

// A batch of query rows handled by one scan/refine launch pair.
//  decode:  unit = (b, kvh); the unit's NQ = g rows are its query heads, all
//           at t = seq_lens[b] - 1.
//  prefill: unit = (b, kvh, block of NP consecutive positions); row r of the
//           unit is head (r % g) at position block*NP + r / g.
struct AttendArgs {
  const void* q;            // [B][Hq][Tq][d]
  int q_host;               // 1: q is mapped page-locked host memory (read over the host link)
  int64_t Tq;               // positions per sequence in q/out (1 for decode)
  int64_t q_begin;          // position of q's first row (prefill)
  const int64_t* seq_lens;  // decode: device [B]; prefill: null
  int64_t pos_lo, pos_hi;   // prefill: q rows [pos_lo, pos_hi) handled by this launch
  int NP;                   // positions per unit (1 for decode)
  const void* K;
  const void* V;
  int64_t sb, sh, st;
  const void* gK;
  const void* gV;
  const int32_t* gCnt;
  const void* pK;
  const void* pV;
  const int32_t* pCnt;
  const int16_t* pBeg;
  const int16_t* gPage;
  const int16_t* perm;
  const void* mK;           // member-ordered key / value copies [..][Cmax * chunk][d]
  const void* mV;
  const int32_t* gMeta;     // size | first page << 16 | end page << 24 per group
  int kv_bits;              // 4: opened pages read from the INT4 codes below
  const uint8_t* qK;        // [..][Cmax * chunk][d / 2] member-ordered 4-bit codes
  const uint8_t* qV;
  const float2* qKs;        // [..][Cmax * P][d] (scale, low) per page slot and channel
  const float2* qVs;
  int B, Hq, Hkv, g;
  int64_t Tmax, Cmax;
  int k, P, G, TP, window, sinks;
  float scale;
  int nsplit;               // splits of each unit's row list (groups, sinks, window)
  int64_t units;            // scan units in this launch
  float* part;              // [units][nsplit][NQ][d+2]  (m, l, acc)
  float2* gsc;              // CUDA-core scan: [units][NQ][Cmax * k] (score, meta) per visible
                            // group: score = scale * q . mean k (-inf: not in that query row's
                            // softmax), meta = the group's gMeta word (as float bits)
  SplitCand* cand;          // tensor-core scan: [units][nsplit][NQ][G] each split's best G
                            // groups per query row (by score, then smaller id); gsc unused
  void* out;                // [B][Hq][Tq][d]
  float* lse;               // [B][Hq][Tq] or null
  int32_t* sel_groups;      // [B][Hq][Tq][G] or null
  int32_t* sel_pages;       // [B][Hq][Tq][G][TP] or null
  uint32_t* status;
};

// TMA tensor maps of the tensor-core scan: group summaries (2-D, rows x d)
// and the KV cache (4-D, d x t x kv-head x sequence), 64 x 128 boxes, 128B swizzle.
struct __align__(64) TcMaps {
  CUtensorMap gK, gV, K, V;
};

// Grouped tensor-core prefill (bf16, d = 128), one wave of query positions
// [w_lo, w_hi) of q at a time.  A wave row is (b * Hq + hq) * NW + (pi - w_lo).
struct PrefillArgs {
  const __nv_bfloat16* q;   // [B][Hq][Tq][d] (device)
  int64_t Tq, q_begin;
  int B, Hq, Hkv, g;
  int64_t Tmax, Cmax;
  int k, P, G, TP, window, sinks;
  float scale_log2;         // softmax scale * log2 e
  const int32_t* gMeta;
  const __nv_bfloat16* gV;
  const int16_t* pBeg;
  const int32_t* pCnt;
  int64_t w_lo, w_hi, NW;   // this wave's q positions; NW = wave rows per (b, hq)
  // workspace
  float* state;             // [rows][132]: m, l (log2 units), -, -, acc[d] (opened groups included)
  int32_t* sel;             // [rows][G] opened group ids, best first, -1 padded
  float* cw;                // [rows][G] weight of the opened group's coarse term, relative to m
  int32_t* pos;             // [rows][G] place of the pair in its group's run
  float* plse;              // [rows][G] pair log-sum-exp (log2 units)
  __nv_bfloat16* po;        // [rows][G][d] pair output (normalised)
  int32_t* list;            // pair ids (row * G + rank) grouped by (unit, group)
  int32_t* list_q;          // beside each: the pair's row of q / out ((b * Hq + hq) * Tq + position)
  int32_t* cnt;             // [Gtot] pairs per (unit, group)
  int32_t* off;             // [Gtot] first pair of each (unit, group)
  int4* items;              // work items {unit * Cmax * k + group, first pair, pairs, 0}: small groups
                            // from items[0], large groups from items[big_items]
  int64_t big_items;
  int32_t* n_items;         // [2] work items of small and of large groups
  int64_t Gtot;             // B * Hkv * Cmax * k
  int item_rows;            // pairs per work item (at most)
  // outputs
  __nv_bfloat16* out;
  float* lse;
  int32_t* sel_groups;
  int32_t* sel_pages;
  uint32_t* status;
};

// TMA tensor maps of the pair kernel: member-ordered K/V copies (32-row
// boxes) and page summaries (16-row boxes), 64 columns, 128B swizzle.
struct __align__(64) PairMaps {
  CUtensorMap mK, mV, pK, pV;
};

cudaError_t launch_prefill_tc_wave(const PrefillArgs& a, const TcMaps& maps, const PairMaps& pmaps, int num_sms,
                                   cudaStream_t stream);
size_t prefill_tc_scan_smem();
size_t prefill_tc_pair_smem();

cudaError_t launch_build(const BuildArgs& a, int dtype, int d, int64_t nchunks, int B,
                         cudaStream_t stream);
cudaError_t launch_append(void* K, void* V, const int64_t* kv_strides_elems, int elem_bytes, int d,
                          const int64_t* seq_lens, const void* kn, const void* vn, int B, int Hkv, int64_t Tmax,
                          cudaStream_t stream);
// maps == nullptr selects the CUDA-core scan; otherwise bf16, d = 128 run the
// tensor-core scan.
cudaError_t launch_attend(const AttendArgs& a, int dtype, int d, int NQ, const TcMaps* maps,
                          cudaStream_t stream);
cudaError_t launch_scan_tc(const AttendArgs& a, const TcMaps& maps, int NQ, cudaStream_t stream);
size_t scan_tc_smem_bytes();

}  // namespace lod
