// rtp_host.h -- host-side helpers shared by the entry points: argument checks,
// head maps and workspace layouts.
#pragma once

#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <utility>

#include "rtp.h"
#include "rtp_common.cuh"

namespace rtp {

constexpr int kDecChunk = 1024;    // tokens per decode scoring / compaction chunk
constexpr int kMaxKeys = 1 << 21;  // composite (score, index) keys use 21 index bits

// Kernel trace: events around each launch while rtp_trace_enable(1) is in force.
void trace_begin(const char* name, cudaStream_t s);
void trace_end(cudaStream_t s);
struct TraceScope {
  cudaStream_t s;
  TraceScope(const char* name, cudaStream_t st) : s(st) { trace_begin(name, st); }
  ~TraceScope() { trace_end(s); }
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline rtp_status check_cuda(cudaError_t e) {
  return e == cudaSuccess ? RTP_OK : RTP_ERR_CUDA;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Launch with programmatic stream serialization: the kernel's CTAs may be
// scheduled while the previous kernel on the stream drains; the kernel itself
// waits (griddep_wait) before it touches anything that kernel wrote.  Inside a
// CUDA graph the edge becomes a programmatic dependency.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                    cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// A [B][L][heads][width] bf16 view: non-null, rows 16-byte aligned.
inline rtp_status check_view(const rtp_view& v, int heads, int width, bool needed) {
  if (!needed) return RTP_OK;
  if (v.ptr == nullptr) return RTP_ERR_INVALID_ARG;
  if (v.stride_l < (int64_t)heads * width || v.stride_b < 0) return RTP_ERR_INVALID_ARG;
  if (!aligned16(v.ptr) || (v.stride_l * 2) % 16 != 0 || (v.stride_b * 2) % 16 != 0)
    return RTP_ERR_ALIGNMENT;
  return RTP_OK;
}

inline rtp_status check_shape(const rtp_shape* s) {
  if (s == nullptr) return RTP_ERR_INVALID_ARG;
  if (s->D != kD) return RTP_ERR_UNSUPPORTED;
  if (s->B < 0 || s->Lq < 0 || s->Lk < 0 || s->H <= 0 || s->Hkv <= 0) return RTP_ERR_INVALID_ARG;
  if (s->H % s->Hkv != 0) return RTP_ERR_INVALID_ARG;
  if (s->H > kMaxHeads) return RTP_ERR_UNSUPPORTED;
  if (s->q_pos0 < 0) return RTP_ERR_INVALID_ARG;
  return RTP_OK;
}

// Causal consistency: every query row's position must have a key row.
inline rtp_status check_causal(const rtp_shape* s) {
  if (s->Lq > 0 && s->q_pos0 + s->Lq - 1 >= (int64_t)s->Lk) return RTP_ERR_INVALID_ARG;
  return RTP_OK;
}

inline rtp_status make_headmap(const rtp_shape* s, const uint8_t* kv_role, int k16_per_kv,
                               HeadMap* hm) {
  if (kv_role == nullptr) return RTP_ERR_INVALID_ARG;
  if (k16_per_kv != 0 && k16_per_kv != 1) return RTP_ERR_INVALID_ARG;
  memset(hm, 0, sizeof(*hm));
  hm->H = s->H;
  hm->Hkv = s->Hkv;
  hm->G = s->H / s->Hkv;
  if (hm->G > 16) return RTP_ERR_UNSUPPORTED;  // decode packs one kv group into 16 mma rows
  for (int g = 0; g < s->Hkv; ++g) {
    if (kv_role[g] > 1) return RTP_ERR_INVALID_ARG;
    if (kv_role[g]) {
      const int rk = hm->n_rkv++;
      hm->rkv[rk] = (int16_t)g;
      for (int j = 0; j < hm->G; ++j) {
        const int hr = hm->n_ret++;
        hm->ret_q[hr] = (int16_t)(g * hm->G + j);
        hm->ret_k16[hr] = (int16_t)(k16_per_kv ? rk : hr);
      }
    } else {
      hm->lkv[hm->n_lkv++] = (int16_t)g;
      hm->n_loc += hm->G;
    }
  }
  hm->H_k16 = k16_per_kv ? hm->n_rkv : hm->n_ret;
  return RTP_OK;
}

// ---------------------------------------------------------------- workspaces
// Every workspace starts with the 256-byte DevStatus block.

// Per-row decode result kept in the workspace.
struct RowRes {
  float t;
  int32_t jtie;
  int32_t count;
  float mass;
};

// Retrieval decode: the per-row top-p state the merge kernel leaves for the
// collection kernel.  Masses are relative to E_top, the upper edge of the row's
// highest occupied score bin.
struct RowSel {
  double T;          // p * Z
  double above;      // mass of the bins above the crossing bin
  double scale_b;    // 2^-21 * exp((bstar + 1) / kappa - E_top): fixed21 -> relative mass
  double Z;
  int32_t bstar;     // absolute score bin holding the cut
  int32_t mode;      // 0 normal, 1 keep all (p >= 1), 2 refine over the stored scores
  uint32_t cnt_above;
  uint32_t n_in;
};

constexpr int kDecWin = 256;           // score bins a scoring CTA keeps per head
constexpr float kDecKappa = 4.0f;      // bins per unit of indexer score
constexpr int kDecGBins = 2048;        // absolute bins per row: scores in [-256, 256)
constexpr int kDecGLo = -1024;         // absolute bin of global bin 0
constexpr int kDecCap = 4096;          // candidates a decode row resolves with one sort
constexpr int kDecMaxSplits = 256;     // split-KV partials per (batch, kv head) in decode
constexpr int kPartRow = kD + 4;       // a partial row: m, l, two pad floats, o[kD] (16-byte rows)

constexpr int kDecSub = 64;            // sub-bins of a row's crossing bin

struct SelectWs {   // prefill top-p selection (select_prefill.cu)
  size_t mask, lists, total;
  int n_sm;
};
SelectWs select_ws_layout();

struct DecodeWs {   // retrieval decode
  size_t scores, hist_m, hist_c, flags, sub_m, sub_c, rowsel, rowres, cand, ncand, counter, list, lcount, loff,
      part, blk, bmask, total;
  int n_chunks, n_splits, Lk_pad, rows, groups;
  int n_blk, n_bwords;  // 64-key blocks per row (of Lk_pad) and their mask words
};

constexpr int kDecBlk = 64;    // keys per block of the block-level top-p
constexpr int kDecHBins = 256; // its histogram bins over the block maxima

inline int decode_list_splits(int groups, int n_chunks) {
  int want = groups > 0 ? (296 + groups - 1) / groups : 1;
  if (want > 4 * n_chunks) want = 4 * n_chunks;  // at least ~256 tokens of list per split
  if (want > kDecMaxSplits) want = kDecMaxSplits;
  return want < 1 ? 1 : want;
}

inline DecodeWs decode_ws_layout(const rtp_shape* s, const HeadMap& hm) {
  DecodeWs w;
  const int64_t N = s->Lk;
  w.n_chunks = (int)((N + kDecChunk - 1) / kDecChunk);
  if (w.n_chunks < 1) w.n_chunks = 1;
  w.Lk_pad = w.n_chunks * kDecChunk;
  w.rows = s->B * hm.n_ret;
  w.groups = s->B * hm.n_rkv;
  w.n_splits = decode_list_splits(w.groups, w.n_chunks);  // largest count any N <= Lk asks for
  const size_t groups = (size_t)w.groups;
  const size_t nc = (size_t)w.n_chunks;
  size_t off = kStatusBytes;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  w.scores = take((size_t)w.rows * w.Lk_pad * 4);
  w.hist_m = take((size_t)w.rows * kDecGBins * 8);   // hist_m, hist_c, flags are one
  w.hist_c = take((size_t)w.rows * kDecGBins * 4);   // contiguous range (cleared per call)
  w.flags = take((size_t)w.rows * 4);
  w.sub_m = take((size_t)w.rows * kDecSub * 8);       // also cleared per call
  w.sub_c = take((size_t)w.rows * kDecSub * 4);
  w.rowsel = take((size_t)w.rows * sizeof(RowSel));
  w.rowres = take((size_t)w.rows * sizeof(RowRes));
  w.cand = take((size_t)w.rows * kDecCap * 8);
  w.ncand = take((size_t)w.rows * 4);
  w.counter = take(groups * 4);
  w.list = take(groups * w.Lk_pad * 8);
  w.lcount = take(groups * nc * 4);
  w.loff = take(groups * (nc + 1) * 4);
  w.part = take(groups * w.n_splits * 16 * kPartRow * 4);
  w.n_blk = w.Lk_pad / kDecBlk;
  w.n_bwords = (w.n_blk + 31) / 32;
  w.blk = take((size_t)w.rows * w.n_blk * 8);       // (max, log-sum-exp) per block
  w.bmask = take((size_t)w.rows * w.n_bwords * 4);  // selected blocks, one bit each
  w.total = off;
  return w;
}

// The retrieval decode's first pass (decode_select.cu): clears the row
// histograms, then scores every key of the cache into the workspace's score
// rows [rows][Lk_pad] and bins them; with block_stats, instead of binning, it
// reduces every 64-key block to (max, log-sum-exp) in the workspace's blk rows.
rtp_status decode_score_pass(const rtp_shape* shape, const HeadMap& hm, int k16_per_kv,
                             const rtp_view& q16, const rtp_view& k16_cache, void* ws,
                             const DecodeWs& L, cudaStream_t s, bool block_stats);

// Buffers the gathered decode attention reads (decode.cu).
struct DecodeLists {
  const uint2* list;       // [groups][Lk_pad], chunk c's entries at c * kDecChunk
  const int32_t* lcount;   // [groups][n_chunks] entries per chunk
  const float* scores;
  const RowRes* rowres;
  float* part;
  int Lk_pad, n_chunks, n_splits;
};

// Static top-k or block-level top-p over the score rows decode_score_pass left
// in the workspace (decode_variants.cu): per-row results, then the kept-key
// union lists for decode_list_attention, described in *lists.
rtp_status decode_variant_select(const rtp_shape* shape, const HeadMap& hm, rtp_select select,
                                 float p, int top_k, void* ws, const DecodeWs& L, float* thr,
                                 int32_t* jtie, int32_t* count, float* mass,
                                 uint32_t* block_mask, DecodeLists* lists, cudaStream_t s);

rtp_status decode_list_attention(const rtp_shape* shape, const HeadMap& hm, const rtp_view& q,
                                 const rtp_view& k, const rtp_view& v, float scale,
                                 const rtp_view& o, float* lse, const DecodeLists& lists,
                                 cudaStream_t s);

struct AttnDecodeWs {  // local / dense decode (range mode)
  size_t part, total;
  int n_splits, keys_per_split;
};

inline AttnDecodeWs range_decode_ws_layout(int64_t n_keys, int groups) {
  AttnDecodeWs w;
  // about two CTAs per SM, at least 64 keys per split
  int64_t want = groups > 0 ? (296 + groups - 1) / groups : 1;
  const int64_t max_splits = (n_keys + 63) / 64;
  if (want > max_splits) want = max_splits;
  if (want > kDecMaxSplits) want = kDecMaxSplits;
  if (want < 1) want = 1;
  int64_t kps = (n_keys + want - 1) / want;
  kps = (kps + 63) / 64 * 64;
  if (kps < 64) kps = 64;
  w.keys_per_split = (int)kps;
  w.n_splits = (int)((n_keys + kps - 1) / kps);
  if (w.n_splits < 1) w.n_splits = 1;
  // sized for `want` splits: a workspace sized for an upper bound on the key
  // count then also fits every smaller key count
  size_t off = kStatusBytes;
  w.part = off;
  off = align_up(off + (size_t)groups * want * 16 * kPartRow * 4, 256);
  w.total = off;
  return w;
}

}  // namespace rtp
