// decode_select.cu -- exact top-p for one decode token per batch entry
// (rtp_sparse_attn_decode): "Dynamic Top-p Selection Mechanism" of the
// paper-graph-ui summary of arXiv 2605.16928, token-exact.
//
// Masses are kept relative to score-bin edges so that no kernel needs the row
// max before it has seen the row: a key with score s sits in the absolute bin
// b = floor(4 s) and contributes exp(s - (b+1)/4) in (0.78, 1] to that bin, as
// 21-bit fixed point.  Integer sums are exact and order-free, so every decision
// below is deterministic.  Per kv group of G retrieval query heads:
//   1. score     stream the k16 cache once (HBM-bound; loaded evict-first, so
//                the score rows stay in L2 for steps 3-5), s = q16 . k16 as one
//                16-term tensor-core dot product (tcgen05, fp32 in TMEM), scores
//                kept in the workspace; each CTA bins its items' scores in shared
//                memory (one 256-bin window per head, 32-bit atomics) and adds
//                the occupied bins into the row's 2048-bin absolute histogram;
//   2. merge     per row: bin masses scaled to the top occupied bin in fp64, Z,
//                T = p Z, the crossing bin and its 64-way sub-bin split;
//   3. collect   per chunk: keys above the crossing bin are kept, keys in it are
//                candidates (collected per row); one ordered list per kv group of
//                every token some head may keep;
//   4. resolve   per row: the crossing sub-bin's candidates, compacted and sorted
//                by (score desc, index asc) by the row's CTA, walked to the exact
//                cut (t, jtie);
//   5. attend    gathered split-KV attention over the lists (decode.cu); the
//                candidate heads are settled there with s > t or (s == t, j <= jtie).
// Rows with scores outside [-256, 256) or more than 4096 keys in the crossing bin
// are resolved by a radix refinement over the stored scores (slower, rare).
#include <algorithm>

#include "dec_bins.cuh"
#include "rtp_host.h"
#include "tcgen05.cuh"
#include "tma.cuh"

namespace rtp {
namespace {

constexpr int kIdxBits = 21;
constexpr unsigned long long kIdxMask = (1ull << kIdxBits) - 1;
constexpr int kKeyBits = 32 + kIdxBits;
constexpr int kThreads = 256;
constexpr double kFix21 = 1.0 / 2097152.0;  // 2^-21
constexpr int kWarpCap = 512;               // candidates one warp sorts on its own

// 2^x for x <= 0 (no subnormal results matter here: x >= -0.37 in every use
// that feeds a decision, and tiny results only need to stay tiny).
__device__ __forceinline__ float ex2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}
// Mass of a key relative to the upper edge (b+1)/kappa of its bin: (0.78, 1].
__device__ __forceinline__ float wbin_f(float s, float bf) {
  const float edge = __fmul_rn(__fadd_rn(bf, 1.0f), 1.0f / kDecKappa);
  return ex2_ftz(__fmul_rn(__fsub_rn(s, edge), kLog2e));
}
__device__ __forceinline__ float wbin(float s, int b) { return wbin_f(s, (float)b); }
// trunc(w * 2^21) for w in [0, 1]: adding 2^23 with rounding toward zero leaves
// the integer part in the low mantissa bits.
__device__ __forceinline__ uint32_t fixed21(float w) {
  return __float_as_uint(__fadd_rz(__fmul_rn(fminf(w, 1.0f), 2097152.0f), 8388608.0f)) -
         0x4B000000u;
}
// Sub-bin of a key inside its (crossing) bin b: 64 equal slices of [b, b+1)/kappa.
__device__ __forceinline__ int subbin(float s, int b) {
  const float frac = __fsub_rn(__fmul_rn(s, kDecKappa), (float)b);
  const int k = (int)__fmul_rn(frac, (float)kDecSub);
  return k < 0 ? 0 : (k > kDecSub - 1 ? kDecSub - 1 : k);
}
// Mass relative to a reference score m (refinement path).
__device__ __forceinline__ float wrel(float s, float m) {
  return exp2f(__fmul_rn(__fsub_rn(s, m), kLog2e));
}
__device__ __forceinline__ unsigned long long comp_key(float s, int j) {
  return ((unsigned long long)score_key(s) << kIdxBits) | (kIdxMask - (unsigned long long)j);
}
__device__ __forceinline__ float key_score(uint32_t key) {
  const uint32_t b = (key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key;
  return __uint_as_float(b);
}

// ------------------------------------------------------------------ 1. score + histogram
// Persistent, TMA-fed, scores on the tensor cores.  Work items are (kv group,
// 512 consecutive keys); a CTA takes a contiguous run of items.  Per 128-key
// sub-tile the producer warp loads the group's kw k16 slots into a ring stage,
// as [128 x 64] four-slot tiles (128-byte swizzled) when kw >= 4, else as kw
// [128 x 16] tiles (32-byte swizzled), both the MMA's K-major layouts,
// and writes the matching [16 x 16] query blocks: slot h's block holds q16 of
// head h in row h (k16 per query head), or the G heads' q16 in rows 0..G-1 (one
// k16 per kv head); every other row stays zero.  The MMA warp issues one
// tcgen05.mma per slot (M = 128, N = 16, K = 16), accumulating
// D[key][head] = q16_head . k16_(key, head's slot) in TMEM: the zero blocks add
// exact zeros, so each score is the 16-term dot product of a single MMA, as in
// the prefill selection.  Consumer warps 0-7 read D, then all 12 per item: the heads'
// max bins, the scores' store, a 256-bin window histogram per head in shared
// memory and its flush into the row's absolute histogram.  Producer and MMA run
// ahead across items, bounded by the ring and by 8 TMEM accumulators.
constexpr int kSItem = 512;                   // keys per work item
constexpr int kSTile = 128;                   // keys per MMA (M)
constexpr int kSN = 16;                       // MMA N: a group's heads, zero-padded
constexpr int kSChunkA = kSTile * kR * 2;     // 4096 B: one slot of a sub-tile
constexpr int kSChunkB = kSN * kR * 2;        // 512 B: one query block
constexpr int kSBufs = 8;                     // TMEM accumulators, kSN columns each
constexpr int kSConsumers = 384;              // 12 warps; warps 0-7 also read TMEM
constexpr int kSProdWarp = kSConsumers / 32, kSMmaWarp = kSProdWarp + 1;
constexpr int kSThreads = kSConsumers + 64;   // + the producer and MMA warps
constexpr int kSRingBytes = 74 * 1024;
constexpr int kSMaxStages = 8;
constexpr uint32_t kSIdesc = idesc_bf16_f32(kSTile, kSN);

struct ScoreParams {
  const uint16_t* q16;
  int64_t q16_sb;
  float* scores;
  unsigned long long* hist_m;  // [rows][kDecGBins]
  uint32_t* hist_c;
  uint32_t* flags;             // [rows]: 1 = a score fell outside the histogram range
  uint32_t* ncand;
  uint32_t* counter;
  DevStatus* status;
  int N, Lk_pad, n_ret, n_rkv, G, lgG, per_kv, rows, groups;
  int kw;            // k16 slots per key of a group: G, or 1 when k16 is per kv head
  int stages;        // ring stages (one sub-tile each)
  int quad;          // 1: kw >= 4, the slots load as four-slot 128-byte-swizzled boxes
  int batch_coord;   // 1, or 0 when every batch entry shares one k16 cache
  int items_per_group, n_items;
  float2* blk;       // block-stats mode: [rows][n_blk] (max, log-sum-exp) of 64-key blocks
  int n_blk;         // (null: the histograms of the exact top-p instead)
};

struct ScoreSmemTail {
  uint64_t full[kSMaxStages];
  uint64_t empty[kSMaxStages];
  uint64_t tfull[kSBufs];
  uint64_t tempty[kSBufs];
  int bgrp[kSMaxStages];  // the group whose query blocks a stage holds (-1: none yet)
  int top[16];
  uint32_t tmem_base;
  int gave_up;
};

// A stage: kw slot tiles, then kw query blocks; 1024-byte multiples.
__host__ __device__ constexpr int score_stage_bytes(int kw) {
  return (kw * (kSChunkA + kSChunkB) + 1023) / 1024 * 1024;
}
__host__ __device__ constexpr int score_stages(int kw) {
  return kSRingBytes / score_stage_bytes(kw) < 2
             ? 2
             : (kSRingBytes / score_stage_bytes(kw) > kSMaxStages
                    ? kSMaxStages
                    : kSRingBytes / score_stage_bytes(kw));
}
__host__ __device__ constexpr size_t score_smem_bytes(int G, int kw) {
  return 1024 + (size_t)score_stages(kw) * score_stage_bytes(kw) +
         (size_t)G * (kSItem + 4) * 4 + (size_t)G * kDecWin * 8 + sizeof(ScoreSmemTail);
}

__global__ void __launch_bounds__(kSThreads, 2)
    dec_score_kernel(const __grid_constant__ CUtensorMap kmap, const ScoreParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int G = p.G, kw = p.kw;
  const int sbytes = score_stage_bytes(kw);
  // stages on a 1024-byte boundary (score_smem_bytes includes the slack)
  unsigned char* ring = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  float* sc = reinterpret_cast<float*>(ring + p.stages * sbytes);         // [G][kSItem+4]
  uint32_t* hm = reinterpret_cast<uint32_t*>(sc + G * (kSItem + 4));     // [G][kDecWin]
  uint32_t* hc = hm + G * kDecWin;
  ScoreSmemTail* tl = reinterpret_cast<ScoreSmemTail*>(hc + G * kDecWin);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // the later kernels of this call count into these
  for (int x = blockIdx.x * kSThreads + tid; x < p.rows; x += gridDim.x * kSThreads)
    p.ncand[x] = 0u;
  for (int x = blockIdx.x * kSThreads + tid; x < p.groups; x += gridDim.x * kSThreads)
    p.counter[x] = 0u;
  for (int x = tid; x < G * kDecWin; x += kSThreads) {
    hm[x] = 0u;
    hc[x] = 0u;
  }
  // query blocks start zero: a group writes only its heads' rows
  for (int s = 0; s < p.stages; ++s)
    for (int x = tid; x < kw * kSChunkB / 16; x += kSThreads)
      *reinterpret_cast<uint4*>(ring + s * sbytes + kw * kSChunkA + x * 16) = make_uint4(0, 0, 0, 0);
  fence_async_smem();
  if (tid == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&tl->full[s], 1);
      mbar_init(&tl->empty[s], 1);
      tl->bgrp[s] = -1;
    }
    for (int i = 0; i < kSBufs; ++i) {
      mbar_init(&tl->tfull[i], 1);
      mbar_init(&tl->tempty[i], 4);  // the four warps that read one accumulator
    }
    tl->gave_up = 0;
    fence_mbar_init();
  }
  if (warp == kSMmaWarp) {
    tmem_alloc(&tl->tmem_base, kSBufs * kSN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tl->tmem_base;
  volatile int* gave_up = &tl->gave_up;
  // a contiguous run of items per CTA: consecutive items share their kv group
  const int per_cta = (p.n_items + (int)gridDim.x - 1) / (int)gridDim.x;
  const int it0 = (int)blockIdx.x * per_cta, it1 = min(it0 + per_cta, p.n_items);

  if (warp == kSProdWarp) {  // ---------------- producer (the whole warp)
    // the k16 stream is read once: evict it first, so that the score rows this
    // kernel writes stay in L2 for the kernels that read them back
    const uint64_t pol = l2_policy_evict_first();
    int stage = 0, n_issued = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int item = it0; ok && item < it1; ++item) {
      const int grp = item / p.items_per_group, j0 = (item % p.items_per_group) * kSItem;
      const int b = grp / p.n_rkv, rk = grp % p.n_rkv;
      const int nvalid = max(0, min(kSItem, p.N - j0));
      const int nsub = (nvalid + kSTile - 1) / kSTile;
      const int slot0 = p.per_kv ? rk : rk * G;
      for (int st = 0; st < nsub; ++st) {
        if (!mbar_wait_warp(&tl->empty[stage], ph ^ 1u, gave_up)) {
          ok = false;
          break;
        }
        unsigned char* sb = ring + stage * sbytes;
        if (tl->bgrp[stage] != grp) {  // this stage's query blocks: the group's q16 rows
          for (int e = lane; e < 2 * G; e += 32) {
            const int h = e >> 1, c = e & 1;  // head, 16-byte half of its row
            const uint4 v = *reinterpret_cast<const uint4*>(p.q16 + b * p.q16_sb +
                                                            (int64_t)(rk * G + h) * kR + c * 8);
            const int blk = p.per_kv ? 0 : h;
            // 32-byte swizzle: the halves of rows 4..7 of every 8 swap
            const int off = h * 32 + ((c ^ ((h >> 2) & 1)) << 4);
            *reinterpret_cast<uint4*>(sb + kw * kSChunkA + blk * kSChunkB + off) = v;
          }
          fence_async_smem();
          __syncwarp();
          if (lane == 0) tl->bgrp[stage] = grp;
          __syncwarp();
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(&tl->full[stage], (uint32_t)(kw * kSChunkA));
          if (p.quad) {  // four slots (128-byte rows) per box
            for (int qd = 0; qd < kw / 4; ++qd)
              tma_load_4d_hint(sb + qd * 4 * kSChunkA, &kmap, 0, slot0 / 4 + qd,
                               j0 + st * kSTile, b * p.batch_coord, &tl->full[stage], pol);
          } else {
            for (int h = 0; h < kw; ++h)
              tma_load_4d_hint(sb + h * kSChunkA, &kmap, 0, slot0 + h, j0 + st * kSTile,
                               b * p.batch_coord, &tl->full[stage], pol);
          }
        }
        ++n_issued;
        if (++stage == p.stages) {
          stage = 0;
          ph ^= 1u;
        }
      }
    }
    if (lane == 0) {
      if (!ok) set_status(p.status, RTP_ERR_DEVICE_TIMEOUT, 20);
      // every copy still in flight lands before the CTA may exit
      for (int k = max(0, n_issued - p.stages); k < n_issued; ++k)
        mbar_wait_drain(&tl->full[k % p.stages], (uint32_t)(k / p.stages) & 1u);
    }
    return;
  }
  if (warp == kSMmaWarp) {  // ---------------- MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t ph = 0, seq = 0;
      bool ok = true;
      for (int item = it0; ok && item < it1; ++item) {
        const int j0 = (item % p.items_per_group) * kSItem;
        const int nsub = (max(0, min(kSItem, p.N - j0)) + kSTile - 1) / kSTile;
        for (int st = 0; st < nsub; ++st) {
          const uint32_t buf = seq % kSBufs;
          if (!mbar_wait(&tl->full[stage], ph, gave_up) ||
              !mbar_wait(&tl->tempty[buf], ((seq / kSBufs) & 1u) ^ 1u, gave_up)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(ring + stage * sbytes);
          for (int h = 0; h < kw; ++h) {
            // slot h: its own 32-byte-swizzled tile, or the 16-element K step h % 4
            // of a 128-byte-swizzled four-slot tile
            const uint64_t adesc =
                p.quad ? sdesc_sw128(sa + (uint32_t)((h >> 2) * 4 * kSChunkA + (h & 3) * 32), 16,
                                     1024)
                       : sdesc_k_sw32(sa + (uint32_t)(h * kSChunkA), 256);
            mma_bf16_ss(tmem + buf * kSN, adesc,
                        sdesc_k_sw32(sa + (uint32_t)(kw * kSChunkA + h * kSChunkB), 256), kSIdesc,
                        h > 0);
          }
          mma_commit(&tl->empty[stage]);  // the stage is free once the MMAs have read it
          mma_commit(&tl->tfull[buf]);    // the accumulator is ready
          ++seq;
          if (++stage == p.stages) {
            stage = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok) set_status(p.status, RTP_ERR_DEVICE_TIMEOUT, 22);
      if (seq > 0)  // the last MMAs are complete before TMEM is released
        mbar_wait_drain(&tl->tfull[(seq - 1) % kSBufs], ((seq - 1) / kSBufs) & 1u);
    }
    __syncwarp();
    tc_fence_before();
    named_bar(2, kSConsumers + 32);  // the consumers are done with TMEM
    tc_fence_after();
    tmem_dealloc(tmem, kSBufs * kSN);
    return;
  }

  // ---------------- consumers (threads 0..kSConsumers-1; named barrier 1)
  const int hh = tid & (G - 1);  // G divides kSConsumers: constant per thread
  uint32_t sub_base = 0;         // sub-tiles of the earlier items (the MMA's sequence)
  bool ok = true;
  for (int item = it0; item < it1; ++item) {
    const int grp = item / p.items_per_group, j0 = (item % p.items_per_group) * kSItem;
    const int b = grp / p.n_rkv, rk = grp % p.n_rkv;
    const int row0 = b * p.n_ret + rk * G;
    const int nvalid = max(0, min(kSItem, p.N - j0));
    const int nsub = (nvalid + kSTile - 1) / kSTile;
    float* scrow = sc + hh * (kSItem + 4);
    // the item's scores: warps 0-3 read sub-tiles 0 and 1, warps 4-7 sub-tiles 2
    // and 3, each its TMEM lane quarter (one key per lane, the heads in columns);
    // keys past N read as -inf
#pragma unroll 1
    for (int u = 0; u < (warp < 8 ? 2 : 0); ++u) {
      const int st = (warp >> 2) * 2 + u;
      const int x = st * kSTile + (warp & 3) * 32 + lane;
      float d[kSN];
      if (st < nsub) {
        const uint32_t seq = sub_base + (uint32_t)st, buf = seq % kSBufs;
        ok = ok && mbar_wait_warp(&tl->tfull[buf], (seq / kSBufs) & 1u, gave_up);
        tc_fence_after();
        if (ok) {
          tmem_ld16(tmem + ((uint32_t)((warp & 3) * 32) << 16) + buf * kSN, d);
        } else {
#pragma unroll
          for (int h = 0; h < kSN; ++h) d[h] = 0.f;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tl->tempty[buf]);
      }
      const bool in = st < nsub && x < nvalid;
#pragma unroll
      for (int h = 0; h < kSN; ++h)
        if (h < G) sc[h * (kSItem + 4) + x] = in ? d[h] + 0.0f : -INFINITY;  // -0 -> +0
    }
    sub_base += (uint32_t)nsub;
    named_bar(1, kSConsumers);
    if (p.blk != nullptr) {  // block-level top-p: (max, log-sum-exp) per 64-key block and head
      const int nblk = (nvalid + 63) / 64;
      for (int task = warp; task < G * nblk; task += kSConsumers / 32) {
        const int h = task / nblk, bi = task % nblk;
        const float* row = sc + h * (kSItem + 4) + bi * 64;
        const float s0 = row[lane], s1 = row[lane + 32];  // keys past N read -inf
        const float mb = warp_max(fmaxf(s0, s1));
        float e = expf(s0 - mb) + expf(s1 - mb);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) e += __shfl_xor_sync(0xffffffffu, e, o);
        if (lane == 0)
          p.blk[(int64_t)(row0 + h) * p.n_blk + j0 / 64 + bi] = make_float2(mb, mb + logf(e));
        float* dst = p.scores + (int64_t)(row0 + h) * p.Lk_pad + j0 + bi * 64;
        dst[lane] = s0;
        dst[lane + 32] = s1;
      }
      named_bar(1, kSConsumers);  // sc is rewritten by the next item
      continue;
    }
    for (int h = warp; h < G; h += kSConsumers / 32) {  // max bin per head, scores' store
      const float* row = sc + h * (kSItem + 4);
      float mx = -INFINITY;
      float* dst = p.scores + (int64_t)(row0 + h) * p.Lk_pad + j0;
      for (int x = lane * 4; x < kSItem; x += 128) {
        const float4 v = *reinterpret_cast<const float4*>(row + x);
        mx = fmaxf(mx, fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w)));
        *reinterpret_cast<float4*>(dst + x) = v;
      }
      mx = warp_max(mx);
      if (lane == 0) tl->top[h] = sbin(mx);
    }
    named_bar(1, kSConsumers);
    // a warp covers 32 / G keys x G heads: bins of different heads never collide
    {
      const int top = tl->top[hh];
      uint32_t* whm = hm + hh * kDecWin;
      uint32_t* whc = hc + hh * kDecWin;
      const int row = row0 + hh;
      const int xs = kSConsumers >> p.lgG;  // keys per pass
      for (int x0 = tid >> p.lgG; x0 < nvalid; x0 += 4 * xs) {
        float m[4], w[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float sv = (x0 + u * xs < nvalid) ? scrow[x0 + u * xs] : -INFINITY;
          m[u] = sbin_m(sv);
          w[u] = sv;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (x0 + u * xs >= nvalid) break;
          const int bi = bin_i(m[u]);
          const int wi = top - bi;  // 0 = the item's top bin
          const uint32_t f = fixed21(wbin_f(w[u], bin_f(m[u])));
          if (wi < kDecWin) {
            atomicAdd(&whm[wi], f);
            atomicAdd(&whc[wi], 1u);
          } else {  // far below this item's max: straight into the row histogram
            int gb = bi - kDecGLo;
            if (gb < 0) {
              gb = 0;
              atomicOr(&p.flags[row], 1u);
            }
            atomicAdd(&p.hist_m[(int64_t)row * kDecGBins + gb], (unsigned long long)f);
            atomicAdd(&p.hist_c[(int64_t)row * kDecGBins + gb], 1u);
          }
        }
      }
    }
    named_bar(1, kSConsumers);
    for (int x = tid; x < G * kDecWin; x += kSConsumers) {  // flush the windows
      const uint32_t c = hc[x];
      if (c == 0) continue;
      const int h = x / kDecWin, wi = x % kDecWin;
      int gb = tl->top[h] - wi - kDecGLo;
      if (gb < 0 || gb >= kDecGBins) {
        gb = gb < 0 ? 0 : kDecGBins - 1;
        atomicOr(&p.flags[row0 + h], 1u);
      }
      atomicAdd(&p.hist_m[(int64_t)(row0 + h) * kDecGBins + gb], (unsigned long long)hm[x]);
      atomicAdd(&p.hist_c[(int64_t)(row0 + h) * kDecGBins + gb], c);
      hm[x] = 0u;
      hc[x] = 0u;
    }
  }
  if (!ok && tid == 0) set_status(p.status, RTP_ERR_DEVICE_TIMEOUT, 21);
  tc_fence_before();
  named_bar(2, kSConsumers + 32);  // TMEM may be released
}

// ------------------------------------------------------------------ 2. per-row merge
struct MergeParams {
  const unsigned long long* hist_m;
  const uint32_t* hist_c;
  const uint32_t* flags;
  RowSel* rowsel;
  float p;
};

constexpr int kBinsPerThread = kDecGBins / kThreads;  // 8

__global__ void __launch_bounds__(kThreads) dec_merge_kernel(const MergeParams p) {
  griddep_wait();  // launched as a dependent of the previous kernel
  __shared__ double wsum[kThreads / 32];
  __shared__ uint32_t wcnt[kThreads / 32];
  __shared__ int s_top;
  __shared__ int s_cross;
  const int row = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // thread t holds the bins t*8 .. t*8+7 counted down from the top bin
  unsigned long long hmv[kBinsPerThread];
  uint32_t hcv[kBinsPerThread];
  int occ = -1;  // highest occupied absolute bin seen by this thread
#pragma unroll
  for (int i = 0; i < kBinsPerThread; ++i) {
    const int gb = kDecGBins - 1 - (tid * kBinsPerThread + i);
    hmv[i] = p.hist_m[(int64_t)row * kDecGBins + gb];
    hcv[i] = p.hist_c[(int64_t)row * kDecGBins + gb];
    if (hcv[i] && occ < 0) occ = gb;
  }
  if (tid == 0) {
    s_top = -1;
    s_cross = 0x7FFFFFFF;
  }
  __syncthreads();
  if (occ >= 0) atomicMax(&s_top, occ);
  __syncthreads();
  const int gtop = s_top < 0 ? 0 : s_top;  // every row has at least one key
  const double etop = (double)(gtop + kDecGLo + 1) / (double)kDecKappa;
  double M[kBinsPerThread];
  double tsum = 0.0;
  uint32_t tcnt = 0;
#pragma unroll
  for (int i = 0; i < kBinsPerThread; ++i) {
    const int gb = kDecGBins - 1 - (tid * kBinsPerThread + i);
    M[i] = hcv[i] ? (double)hmv[i] * kFix21 *
                        exp((double)(gb + kDecGLo + 1) / (double)kDecKappa - etop)
                  : 0.0;
    tsum += M[i];
    tcnt += hcv[i];
  }
  // fixed-order scans over threads (bins in descending order)
  double incl = tsum;
  uint32_t cincl = tcnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double y = __shfl_up_sync(0xffffffffu, incl, o);
    const uint32_t cy = __shfl_up_sync(0xffffffffu, cincl, o);
    if (lane >= o) {
      incl += y;
      cincl += cy;
    }
  }
  if (lane == 31) {
    wsum[warp] = incl;
    wcnt[warp] = cincl;
  }
  __syncthreads();
  double before = 0.0, Z = 0.0;
  uint32_t cbefore = 0;
  for (int w = 0; w < kThreads / 32; ++w) {
    if (w < warp) {
      before += wsum[w];
      cbefore += wcnt[w];
    }
    Z += wsum[w];
  }
  before += incl - tsum;
  cbefore += cincl - tcnt;
  const double T = (double)p.p * Z;
  // this thread's bins: the first one where the running mass reaches T
  double acc = before;
  int my_cross = 0x7FFFFFFF;
  double my_above = 0.0;
  uint32_t my_cnt = 0, my_nin = 0;
  uint32_t c = cbefore;
#pragma unroll
  for (int i = 0; i < kBinsPerThread; ++i) {
    if (hcv[i] && my_cross == 0x7FFFFFFF && acc + M[i] >= T) {
      my_cross = tid * kBinsPerThread + i;
      my_above = acc;
      my_cnt = c;
      my_nin = hcv[i];
    }
    acc += M[i];
    c += hcv[i];
  }
  if (my_cross != 0x7FFFFFFF) atomicMin(&s_cross, my_cross);
  __syncthreads();
  const int cross = s_cross;
  const bool flagged = p.flags[row] != 0;
  if (cross != 0x7FFFFFFF && my_cross == cross) {
    RowSel rs;
    rs.bstar = (kDecGBins - 1 - cross) + kDecGLo;
    rs.T = T;
    rs.Z = Z;
    rs.above = my_above;
    rs.cnt_above = my_cnt;
    rs.n_in = my_nin;
    rs.scale_b = kFix21 * exp((double)(rs.bstar + 1) / (double)kDecKappa - etop);
    rs.mode = (p.p >= 1.f) ? 1 : ((flagged || rs.n_in > (uint32_t)kDecCap) ? 2 : 0);
    p.rowsel[row] = rs;
  }
  if (cross == 0x7FFFFFFF && tid == 0) {  // T out of reach by rounding, or p >= 1
    RowSel rs;
    rs.bstar = kDecGLo - 1;
    rs.T = T;
    rs.Z = Z;
    rs.above = 0.0;
    rs.cnt_above = 0;
    rs.n_in = 0;
    rs.scale_b = 0.0;
    rs.mode = (p.p >= 1.f) ? 1 : 2;
    p.rowsel[row] = rs;
  }
}

// ------------------------------------------------------------------ 3. collect + compact + cut
struct CollectParams {
  const float* scores;
  const RowSel* rowsel;
  unsigned long long* sub_m;  // [rows][kDecSub]: the crossing bin split 64 ways
  uint32_t* sub_c;
  unsigned long long* cand;  // [rows][kDecCap]
  uint32_t* ncand;
  uint2* list;               // [groups][Lk_pad]
  int32_t* lcount;           // [groups][nc]
  int32_t* loff;             // [groups][nc + 1]
  uint32_t* counter;
  RowRes* rowres;
  float* thr;
  int32_t* jtie;
  int32_t* count;
  float* mass;
  DevStatus* status;
  int N, Lk_pad, nc, n_ret, n_rkv, G;
  float p;
};

struct CollectSmem {
  RowSel rs[16];
  float lo[16], hi[16];  // the crossing bin's edges bstar / kappa, (bstar + 1) / kappa
  int wsum[kThreads / 32];
};

struct ResolveSmem {
  unsigned long long wc[kWarpCap];  // warp-sorted candidates
  unsigned long long cand[kDecCap]; // block-wide candidates
  unsigned long long tsum[kThreads];
  unsigned long long hm[256];
  uint32_t hc[256];
  unsigned long long red[kThreads / 32];
  int ncand;
  int cut;
  unsigned long long s_acc;
  uint32_t s_cnt, s_nin;
  int s_k;
};

__device__ unsigned long long block_sum_u64(unsigned long long v, unsigned long long* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const uint32_t lo = __shfl_xor_sync(0xffffffffu, (uint32_t)v, o);
    const uint32_t hi = __shfl_xor_sync(0xffffffffu, (uint32_t)(v >> 32), o);
    v += ((unsigned long long)hi << 32) | lo;
  }
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  unsigned long long s = 0;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) s += red[w];
  __syncthreads();
  return s;
}

// Bitonic sort of a[0..n) descending (padded with zeros to a power of two), one block.
__device__ void sort_desc_block(unsigned long long* a, int n) {
  int n2 = 1;
  while (n2 < n) n2 <<= 1;
  for (int i = n + threadIdx.x; i < n2; i += blockDim.x) a[i] = 0ull;
  __syncthreads();
  for (int k = 2; k <= n2; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < n2; i += blockDim.x) {
        const int l = i ^ j;
        if (l > i) {
          const bool desc = (i & k) == 0;
          const unsigned long long x = a[i], y = a[l];
          if (desc ? (x < y) : (x > y)) {
            a[i] = y;
            a[l] = x;
          }
        }
      }
      __syncthreads();
    }
  }
}

// The same, one warp.
// 32 keys, one per lane, sorted descending across the warp (bitonic, in registers):
// lane i returns the i-th largest.
__device__ __forceinline__ unsigned long long sort32_desc(unsigned long long v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1)
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      const uint32_t lo = __shfl_xor_sync(0xffffffffu, (uint32_t)v, j);
      const uint32_t hi = __shfl_xor_sync(0xffffffffu, (uint32_t)(v >> 32), j);
      const unsigned long long o = ((unsigned long long)hi << 32) | lo;
      // the pair's lower lane keeps the larger key in a descending block
      const bool desc = (lane & k) == 0, lower = (lane & j) == 0;
      v = (lower == desc) ? (v > o ? v : o) : (v < o ? v : o);
    }
  return v;
}

__device__ void sort_desc_warp(unsigned long long* a, int n) {
  const int lane = threadIdx.x & 31;
  int n2 = 1;
  while (n2 < n) n2 <<= 1;
  for (int i = n + lane; i < n2; i += 32) a[i] = 0ull;
  __syncwarp();
  for (int k = 2; k <= n2; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = lane; i < n2; i += 32) {
        const int l = i ^ j;
        if (l > i) {
          const bool desc = (i & k) == 0;
          const unsigned long long x = a[i], y = a[l];
          if (desc ? (x < y) : (x > y)) {
            a[i] = y;
            a[l] = x;
          }
        }
      }
      __syncwarp();
    }
  }
}

// Walk the sorted candidates a[0..n) of a normal row with one warp: the first k
// with above + scale * sum_{a<=k} fixed21(w(a)) >= T.  Lane 0 returns the result.
__device__ RowRes warp_walk(const unsigned long long* a, int n, const RowSel& rs) {
  const int lane = threadIdx.x & 31;
  const int per = (n + 31) / 32;
  const int a0 = lane * per, a1 = min(n, a0 + per);
  unsigned long long seg = 0;
  for (int i = a0; i < a1; ++i)
    seg += fixed21(wbin(key_score((uint32_t)(a[i] >> kIdxBits)), rs.bstar));
  unsigned long long incl = seg;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t lo = __shfl_up_sync(0xffffffffu, (uint32_t)incl, o);
    const uint32_t hi = __shfl_up_sync(0xffffffffu, (uint32_t)(incl >> 32), o);
    if (lane >= o) incl += ((unsigned long long)hi << 32) | lo;
  }
  unsigned long long cum = incl - seg;
  int my = 0x7FFFFFFF;
  unsigned long long mycum = 0;
  for (int i = a0; i < a1; ++i) {
    cum += fixed21(wbin(key_score((uint32_t)(a[i] >> kIdxBits)), rs.bstar));
    if (rs.above + (double)cum * rs.scale_b >= rs.T) {
      my = i;
      mycum = cum;
      break;
    }
  }
  int cut = my;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cut = min(cut, __shfl_xor_sync(0xffffffffu, cut, o));
  unsigned long long cutcum;
  if (cut == 0x7FFFFFFF) {  // rounding kept T out of reach: keep every candidate
    cut = n - 1;
    cutcum = __shfl_sync(0xffffffffu, incl, 31);
  } else {
    const unsigned ball = __ballot_sync(0xffffffffu, my == cut);
    const int src = __ffs(ball) - 1;
    const uint32_t lo = __shfl_sync(0xffffffffu, (uint32_t)mycum, src);
    const uint32_t hi = __shfl_sync(0xffffffffu, (uint32_t)(mycum >> 32), src);
    cutcum = ((unsigned long long)hi << 32) | lo;
  }
  RowRes out;
  const unsigned long long ck = a[cut];
  out.t = key_score((uint32_t)(ck >> kIdxBits));
  out.jtie = (int32_t)(kIdxMask - (ck & kIdxMask));
  out.count = (int32_t)(rs.cnt_above + cut + 1);
  out.mass = (float)((rs.above + (double)cutcum * rs.scale_b) / rs.Z);
  return out;
}

// Block-wide walk for rows with more than kWarpCap candidates.
template <class F>
__device__ int walk_cut(ResolveSmem& sm, int n, F&& fmass, double base, double scale, double T,
                        unsigned long long& cum_out) {
  const int tid = threadIdx.x;
  const int per = (n + kThreads - 1) / kThreads;
  const int a0 = tid * per, a1 = min(n, a0 + per);
  unsigned long long seg = 0;
  for (int a = a0; a < a1; ++a) seg += fmass(a);
  sm.tsum[tid] = seg;
  if (tid == 0) sm.cut = 0x7FFFFFFF;
  __syncthreads();
  unsigned long long before = 0;
  for (int q = 0; q < tid; ++q) before += sm.tsum[q];
  unsigned long long cum = before;
  for (int a = a0; a < a1; ++a) {
    cum += fmass(a);
    if (base + (double)cum * scale >= T) {
      atomicMin(&sm.cut, a);
      break;
    }
  }
  __syncthreads();
  int cut = sm.cut;
  if (cut == 0x7FFFFFFF) cut = n - 1;
  if (tid == 0) {
    unsigned long long c2 = 0;
    for (int a = 0; a <= cut; ++a) c2 += fmass(a);
    sm.tsum[0] = c2;
  }
  __syncthreads();
  cum_out = sm.tsum[0];
  __syncthreads();
  return cut;
}

// Exact cut of one row by radix refinement over all its stored scores (masses
// relative to the row max, composite (score, index) keys, 8-bit digits).  One CTA.
__device__ void refine_row(ResolveSmem& sm, const CollectParams& p, const float* srow,
                           RowRes& out) {
  const int tid = threadIdx.x;
  const int N = p.N;
  float mx = -INFINITY;
  for (int j = tid; j < N; j += kThreads) mx = fmaxf(mx, srow[j]);
  mx = warp_max(mx);
  __syncthreads();
  if ((tid & 31) == 0) sm.tsum[tid >> 5] = (unsigned long long)__float_as_uint(mx);
  __syncthreads();
  float m = -INFINITY;
  for (int w = 0; w < kThreads / 32; ++w) m = fmaxf(m, __uint_as_float((uint32_t)sm.tsum[w]));
  __syncthreads();
  unsigned long long z = 0;
  for (int j = tid; j < N; j += kThreads) z += mass_fixed40(wrel(srow[j], m));
  const unsigned long long Z = block_sum_u64(z, sm.red);
  const double T = (double)p.p * (double)Z;
  int pb = 0;
  unsigned long long prefix = 0, acc_above = 0;
  uint32_t cnt_above = 0, n_in = (uint32_t)N;
  auto member = [&](float s, int j, unsigned long long& ck) -> bool {
    ck = comp_key(s, j);
    return pb == 0 || (ck >> (kKeyBits - pb)) == prefix;
  };
  for (int lvl = 0; lvl < 8 && n_in > (uint32_t)kDecCap && pb < kKeyBits; ++lvl) {
    const int w = min(8, kKeyBits - pb);
    for (int bb = tid; bb < 256; bb += kThreads) {
      sm.hm[bb] = 0;
      sm.hc[bb] = 0;
    }
    __syncthreads();
    for (int j = tid; j < N; j += kThreads) {
      const float s = srow[j];
      unsigned long long ck;
      if (!member(s, j, ck)) continue;
      const int digit = (int)((ck >> (kKeyBits - pb - w)) & ((1ull << w) - 1));
      atomicAdd(&sm.hm[(1 << w) - 1 - digit], mass_fixed40(wrel(s, m)));
      atomicAdd(&sm.hc[(1 << w) - 1 - digit], 1u);
    }
    __syncthreads();
    if (tid == 0) {
      unsigned long long a = acc_above;
      uint32_t c = cnt_above, nin = 0;
      int last = -1, k = -1;
      for (int bb = 0; bb < (1 << w); ++bb) {
        if (sm.hc[bb] == 0) continue;
        last = bb;
        if ((double)(a + sm.hm[bb]) >= T) {
          k = bb;
          nin = sm.hc[bb];
          break;
        }
        a += sm.hm[bb];
        c += sm.hc[bb];
      }
      if (k < 0) {
        k = last;
        a -= sm.hm[last];
        c -= sm.hc[last];
        nin = sm.hc[last];
      }
      sm.s_acc = a;
      sm.s_cnt = c;
      sm.s_nin = nin;
      sm.s_k = (1 << w) - 1 - k;
    }
    __syncthreads();
    acc_above = sm.s_acc;
    cnt_above = sm.s_cnt;
    n_in = sm.s_nin;
    prefix = (prefix << w) | (unsigned long long)sm.s_k;
    pb += w;
    __syncthreads();
  }
  if (tid == 0) sm.ncand = 0;
  __syncthreads();
  for (int j = tid; j < N; j += kThreads) {
    unsigned long long ck;
    if (!member(srow[j], j, ck)) continue;
    const int idx = atomicAdd(&sm.ncand, 1);
    if (idx < kDecCap) sm.cand[idx] = ck;
  }
  __syncthreads();
  int n = min(sm.ncand, kDecCap);
  if (sm.ncand > kDecCap && tid == 0) set_status(p.status, RTP_ERR_DEVICE_TIMEOUT, 31);
  sort_desc_block(sm.cand, n);
  unsigned long long cum = 0;
  const int cut = walk_cut(
      sm, n,
      [&](int a) {
        return mass_fixed40(wrel(key_score((uint32_t)(sm.cand[a] >> kIdxBits)), m));
      },
      (double)acc_above, 1.0, T, cum);
  const unsigned long long ck = sm.cand[cut];
  out.t = key_score((uint32_t)(ck >> kIdxBits));
  out.jtie = (int32_t)(kIdxMask - (ck & kIdxMask));
  out.count = (int32_t)(cnt_above + cut + 1);
  out.mass = (float)((double)(acc_above + cum) / (double)Z);
}

// A normal row whose crossing bin holds more than kWarpCap keys: radix levels
// over the candidates' composite keys (in shared memory) narrow the crossing down
// to a few keys, which warp 0 sorts and walks.  Block-wide.
__device__ RowRes resolve_many(ResolveSmem& sm, const CollectParams& p, int row, RowSel rs,
                               int n) {
  const int tid = threadIdx.x;
  for (int a = tid; a < n; a += kThreads) sm.cand[a] = __ldcg(&p.cand[(int64_t)row * kDecCap + a]);
  __syncthreads();
  // common prefix of every candidate key
  unsigned long long kmin = ~0ull, kmax = 0ull;
  for (int a = tid; a < n; a += kThreads) {
    kmin = min(kmin, sm.cand[a]);
    kmax = max(kmax, sm.cand[a]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
  }
  if ((tid & 31) == 0) {
    sm.tsum[tid >> 5] = kmin;
    sm.tsum[8 + (tid >> 5)] = kmax;
  }
  __syncthreads();
  kmin = ~0ull;
  kmax = 0ull;
  for (int w = 0; w < kThreads / 32; ++w) {
    kmin = min(kmin, sm.tsum[w]);
    kmax = max(kmax, sm.tsum[8 + w]);
  }
  __syncthreads();
  int pb = (kmin == kmax) ? kKeyBits : (__clzll(kmin ^ kmax) - (64 - kKeyBits));
  unsigned long long prefix = pb > 0 ? (kmax >> (kKeyBits - pb)) : 0ull;
  unsigned long long base = 0;  // fixed21 mass of candidates above the current range
  uint32_t cbase = 0;
  uint32_t n_in = (uint32_t)n;
  auto member = [&](unsigned long long ck) {
    return pb == 0 || (ck >> (kKeyBits - pb)) == prefix;
  };
  for (int lvl = 0; lvl < 8 && n_in > (uint32_t)kWarpCap && pb < kKeyBits; ++lvl) {
    const int w = min(8, kKeyBits - pb);
    for (int bb = tid; bb < 256; bb += kThreads) {
      sm.hm[bb] = 0;
      sm.hc[bb] = 0;
    }
    __syncthreads();
    for (int a = tid; a < n; a += kThreads) {
      const unsigned long long ck = sm.cand[a];
      if (!member(ck)) continue;
      const int digit = (int)((ck >> (kKeyBits - pb - w)) & ((1ull << w) - 1));
      atomicAdd(&sm.hm[(1 << w) - 1 - digit],
                (unsigned long long)fixed21(wbin(key_score((uint32_t)(ck >> kIdxBits)), rs.bstar)));
      atomicAdd(&sm.hc[(1 << w) - 1 - digit], 1u);
    }
    __syncthreads();
    if (tid == 0) {
      unsigned long long a = base;
      uint32_t c = cbase, nin = 0;
      int last = -1, k = -1;
      for (int bb = 0; bb < (1 << w); ++bb) {
        if (sm.hc[bb] == 0) continue;
        last = bb;
        if (rs.above + (double)(a + sm.hm[bb]) * rs.scale_b >= rs.T) {
          k = bb;
          nin = sm.hc[bb];
          break;
        }
        a += sm.hm[bb];
        c += sm.hc[bb];
      }
      if (k < 0) {
        k = last;
        a -= sm.hm[last];
        c -= sm.hc[last];
        nin = sm.hc[last];
      }
      sm.s_acc = a;
      sm.s_cnt = c;
      sm.s_nin = nin;
      sm.s_k = (1 << w) - 1 - k;
    }
    __syncthreads();
    base = sm.s_acc;
    cbase = sm.s_cnt;
    n_in = sm.s_nin;
    prefix = (prefix << w) | (unsigned long long)sm.s_k;
    pb += w;
    __syncthreads();
  }
  // the remaining candidates -> warp 0
  if (tid == 0) sm.ncand = 0;
  __syncthreads();
  for (int a = tid; a < n; a += kThreads) {
    const unsigned long long ck = sm.cand[a];
    if (!member(ck)) continue;
    const int idx = atomicAdd(&sm.ncand, 1);
    if (idx < kWarpCap) sm.wc[idx] = ck;
  }
  __syncthreads();
  RowRes rr;
  if (tid < 32) {
    const int m = min(sm.ncand, kWarpCap);
    if (sm.ncand > kWarpCap && tid == 0) set_status(p.status, RTP_ERR_DEVICE_TIMEOUT, 33);
    RowSel r2 = rs;
    r2.above = rs.above + (double)base * rs.scale_b;
    r2.cnt_above = rs.cnt_above + cbase;
    sort_desc_warp(sm.wc, m);
    rr = warp_walk(sm.wc, m, r2);
    // the walk's mass counts only the narrowed keys; add the candidates above them
  }
  __syncthreads();
  return rr;
}


__global__ void __launch_bounds__(kThreads, 8) dec_collect_kernel(const CollectParams p) {
  griddep_wait();  // launched as a dependent of the previous kernel
  extern __shared__ __align__(16) unsigned char smem_raw[];
  CollectSmem& sm = *reinterpret_cast<CollectSmem*>(smem_raw);
  const int chunk = blockIdx.x, grp = blockIdx.y;
  const int b = grp / p.n_rkv, rk = grp % p.n_rkv;
  const int tid = threadIdx.x;
  const int G = p.G;
  const int row0 = b * p.n_ret + rk * G;
  if (tid < G) {
    const RowSel rs = p.rowsel[row0 + tid];
    sm.rs[tid] = rs;
    // sbin(s) = floor(kappa s) on exact multiples of 1 / kappa, clamped far outside
    // the histogram's range: sbin(s) > bstar iff s >= hi, sbin(s) == bstar iff
    // lo <= s < hi (NaN is neither, as sbin puts it at the bottom)
    sm.lo[tid] = (float)rs.bstar * (1.0f / kDecKappa);
    sm.hi[tid] = (float)(rs.bstar + 1) * (1.0f / kDecKappa);
  }
  __syncthreads();
  const int j0 = chunk * kDecChunk + tid * 4;
  bool valid[4];  // keys past N are skipped
#pragma unroll
  for (int e = 0; e < 4; ++e) valid[e] = j0 + e < p.N;
  uint32_t keep[4] = {0, 0, 0, 0}, cand[4] = {0, 0, 0, 0};
  for (int h = 0; h < G; ++h) {
    const int mode = sm.rs[h].mode;  // the same for every thread of the CTA
    const float4 v =
        *reinterpret_cast<const float4*>(p.scores + (int64_t)(row0 + h) * p.Lk_pad + j0);
    const float vs[4] = {v.x, v.y, v.z, v.w};
    if (mode != 0) {  // 1: every key kept; 2: settled per key by the attention kernel
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (valid[e]) (mode == 1 ? keep[e] : cand[e]) |= 1u << h;
      continue;
    }
    const float lo = sm.lo[h], hi = sm.hi[h];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (!valid[e]) continue;
      const int j = j0 + e;
      if (vs[e] >= hi) {
        keep[e] |= 1u << h;
      } else if (vs[e] >= lo) {
        const RowSel& rs = sm.rs[h];
        cand[e] |= 1u << h;
        const uint32_t idx = atomicAdd(&p.ncand[row0 + h], 1u);
        if (idx < (uint32_t)kDecCap)
          p.cand[(int64_t)(row0 + h) * kDecCap + idx] = comp_key(vs[e], j);
        const int sb = subbin(vs[e], rs.bstar);
        atomicAdd(&p.sub_m[(int64_t)(row0 + h) * kDecSub + sb],
                  (unsigned long long)fixed21(wbin(vs[e], rs.bstar)));
        atomicAdd(&p.sub_c[(int64_t)(row0 + h) * kDecSub + sb], 1u);
      }
    }
  }
  // ordered compaction of the tokens some head may keep
  const int lane = tid & 31, warp = tid >> 5;
  int cnt = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e) cnt += (keep[e] | cand[e]) != 0;
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) sm.wsum[warp] = incl;
  __syncthreads();
  int off = incl - cnt;
  for (int w = 0; w < warp; ++w) off += sm.wsum[w];
  uint2* dst = p.list + (int64_t)grp * p.Lk_pad + chunk * kDecChunk;
#pragma unroll
  for (int e = 0; e < 4; ++e)
    if (keep[e] | cand[e]) dst[off++] = make_uint2((uint32_t)(j0 + e), keep[e] | (cand[e] << 16));
  if (tid == kThreads - 1) {
    int tot = 0;
    for (int w = 0; w < kThreads / 32; ++w) tot += sm.wsum[w];
    p.lcount[(int64_t)grp * p.nc + chunk] = tot;
  }
}

// One CTA per retrieval row: the exact cut inside the crossing bin.
__global__ void __launch_bounds__(kThreads) dec_resolve_kernel(const CollectParams p) {
  griddep_wait();  // launched as a dependent of the previous kernel
  extern __shared__ __align__(16) unsigned char smem_raw[];
  ResolveSmem& sm = *reinterpret_cast<ResolveSmem*>(smem_raw);
  const int row = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31;
  // the row's first kThreads candidate slots, loaded with its descriptor (the
  // slots past the count are read but unused; the row has kDecCap of them)
  const unsigned long long ck_pre = __ldcg(p.cand + (int64_t)row * kDecCap + tid);
  const RowSel rs = p.rowsel[row];
  RowRes rr;
  if (rs.mode == 1) {
    rr.t = -INFINITY;
    rr.jtie = p.N - 1;
    rr.count = p.N;
    rr.mass = 1.f;
  } else {
    const int n = (int)min(p.ncand[row], (uint32_t)kDecCap);
    // crossing sub-bin (warp 0): sub-bins from the top, masses in fixed21 units
    if (tid < 32 && rs.mode == 0 && n > 0) {
      const unsigned long long m0 = p.sub_m[(int64_t)row * kDecSub + (kDecSub - 1 - 2 * lane)];
      const unsigned long long m1 = p.sub_m[(int64_t)row * kDecSub + (kDecSub - 2 - 2 * lane)];
      const uint32_t n0 = p.sub_c[(int64_t)row * kDecSub + (kDecSub - 1 - 2 * lane)];
      const uint32_t n1 = p.sub_c[(int64_t)row * kDecSub + (kDecSub - 2 - 2 * lane)];
      unsigned long long incl = m0 + m1;
      uint32_t cincl = n0 + n1;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t lo = __shfl_up_sync(0xffffffffu, (uint32_t)incl, o);
        const uint32_t hi = __shfl_up_sync(0xffffffffu, (uint32_t)(incl >> 32), o);
        const uint32_t cy = __shfl_up_sync(0xffffffffu, cincl, o);
        if (lane >= o) {
          incl += ((unsigned long long)hi << 32) | lo;
          cincl += cy;
        }
      }
      unsigned long long a = incl - m0 - m1;
      uint32_t c = cincl - n0 - n1;
      int my = 0x7FFFFFFF;
      unsigned long long my_a = 0;
      uint32_t my_c = 0, my_n = 0;
      if (n0 && rs.above + (double)(a + m0) * rs.scale_b >= rs.T) {
        my = 2 * lane; my_a = a; my_c = c; my_n = n0;
      } else if (n1 && rs.above + (double)(a + m0 + m1) * rs.scale_b >= rs.T) {
        my = 2 * lane + 1; my_a = a + m0; my_c = c + n0; my_n = n1;
      }
      int cut = my;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) cut = min(cut, __shfl_xor_sync(0xffffffffu, cut, o));
      if (cut == my && my != 0x7FFFFFFF) {
        sm.s_acc = my_a;
        sm.s_cnt = my_c;
        sm.s_nin = my_n;
        sm.s_k = kDecSub - 1 - cut;  // the sub-bin index
      }
      if (cut == 0x7FFFFFFF && lane == 0) sm.s_k = -1;
    }
    __syncthreads();
    const int ksub = (rs.mode == 0 && n > 0) ? sm.s_k : -1;
    if (ksub >= 0 && sm.s_nin <= (uint32_t)kWarpCap) {
      RowSel r2 = rs;
      r2.above = rs.above + (double)sm.s_acc * rs.scale_b;
      r2.cnt_above = rs.cnt_above + sm.s_cnt;
      // the candidates of the crossing sub-bin, compacted by the block in order
      const unsigned long long* src = p.cand + (int64_t)row * kDecCap;
      int m = 0;
      for (int i0 = 0; i0 < n; i0 += kThreads) {
        const int i = i0 + tid;
        unsigned long long ck = 0;
        bool in = false;
        if (i < n) {
          ck = i0 == 0 ? ck_pre : __ldcg(src + i);
          in = subbin(key_score((uint32_t)(ck >> kIdxBits)), rs.bstar) == ksub;
        }
        const unsigned ball = __ballot_sync(0xffffffffu, in);
        if (lane == 0) sm.hc[tid >> 5] = __popc(ball);
        __syncthreads();
        int off = m;
        for (int w2 = 0; w2 < (tid >> 5); ++w2) off += (int)sm.hc[w2];
        if (in) sm.wc[off + __popc(ball & ((1u << lane) - 1u))] = ck;
        for (int w2 = 0; w2 < kThreads / 32; ++w2) m += (int)sm.hc[w2];
        __syncthreads();
      }
      if (m <= 32) {  // one warp: a register sort, no block barriers
        if (tid < 32) {
          sm.wc[lane] = sort32_desc(lane < m ? sm.wc[lane] : 0ull);
          __syncwarp();
          rr = warp_walk(sm.wc, m, r2);
        }
      } else {
        sort_desc_block(sm.wc, m);
        if (tid < 32) rr = warp_walk(sm.wc, m, r2);
      }
    } else if (rs.mode == 0 && n > 0 && n <= kWarpCap) {
      for (int i = tid; i < n; i += kThreads) sm.wc[i] = __ldcg(p.cand + (int64_t)row * kDecCap + i);
      __syncthreads();
      sort_desc_block(sm.wc, n);
      if (tid < 32) rr = warp_walk(sm.wc, n, rs);
    } else if (rs.mode == 0 && n > 0) {
      rr = resolve_many(sm, p, row, rs, n);
    } else {
      refine_row(sm, p, p.scores + (int64_t)row * p.Lk_pad, rr);
    }
  }
  if (tid == 0) {
    p.rowres[row] = rr;
    if (p.thr) p.thr[row] = rr.t;
    if (p.jtie) p.jtie[row] = rr.jtie;
    if (p.count) p.count[row] = rr.count;
    if (p.mass) p.mass[row] = rr.mass;
  }
}

}  // namespace
}  // namespace rtp

using namespace rtp;

namespace rtp {
rtp_status decode_score_pass(const rtp_shape* shape, const HeadMap& hm, int k16_per_kv_head,
                             const rtp_view& q16, const rtp_view& k16_cache, void* ws,
                             const DecodeWs& L, cudaStream_t s, bool block_stats) {
  rtp_status st = RTP_OK;
  char* w = static_cast<char*>(ws);
  const int N = (int)(shape->q_pos0 + 1);  // keys 0..P
  const int groups = shape->B * hm.n_rkv;
  auto at = [&](size_t off) { return static_cast<void*>(w + off); };
  // the row histograms and flags accumulate with atomics: clear them
  if (cudaMemsetAsync(at(L.hist_m), 0, L.rowsel - L.hist_m, s) != cudaSuccess)
    return RTP_ERR_CUDA;
  {  // 1. scores + histograms
    ScoreParams sp;
    sp.q16 = static_cast<const uint16_t*>(q16.ptr);
    sp.q16_sb = q16.stride_b;
    sp.scores = static_cast<float*>(at(L.scores));
    sp.hist_m = static_cast<unsigned long long*>(at(L.hist_m));
    sp.hist_c = static_cast<uint32_t*>(at(L.hist_c));
    sp.flags = static_cast<uint32_t*>(at(L.flags));
    sp.ncand = static_cast<uint32_t*>(at(L.ncand));
    sp.counter = static_cast<uint32_t*>(at(L.counter));
    sp.status = static_cast<DevStatus*>(ws);
    sp.N = N;
    sp.Lk_pad = L.Lk_pad;
    sp.n_ret = hm.n_ret;
    sp.n_rkv = hm.n_rkv;
    sp.G = hm.G;
    sp.lgG = 0;
    while ((1 << sp.lgG) < hm.G) ++sp.lgG;  // G is a power of two (it divides 256)
    sp.per_kv = k16_per_kv_head;
    sp.rows = L.rows;
    sp.groups = groups;
    sp.kw = k16_per_kv_head ? 1 : hm.G;
    sp.stages = score_stages(sp.kw);
    sp.quad = sp.kw >= 4 ? 1 : 0;  // kw >= 4: group slots start at a multiple of 4
    sp.batch_coord = (k16_cache.stride_b != 0 || shape->B == 1) ? 1 : 0;
    sp.items_per_group = L.Lk_pad / kSItem;
    sp.n_items = groups * sp.items_per_group;
    sp.blk = block_stats ? static_cast<float2*>(at(L.blk)) : nullptr;
    sp.n_blk = L.n_blk;
    // k16 as a 4-D tensor {16 x slots per box, slot boxes, keys 0..N-1, batch}
    // (keys past N read as 0); boxes of 128 keys x one slot (32-byte swizzled) or
    // x four slots (128-byte swizzled)
    CUtensorMap kmap;
    const uint64_t sl_bytes = (uint64_t)k16_cache.stride_l * 2;
    const uint64_t sb_bytes =
        sp.batch_coord && k16_cache.stride_b != 0 ? (uint64_t)k16_cache.stride_b * 2 : sl_bytes * N;
    const uint64_t nbatch = sp.batch_coord ? (uint64_t)shape->B : 1u;
    const uint64_t dims[4] = {sp.quad ? 64u : 16u,
                              (uint64_t)hm.H_k16 / (sp.quad ? 4u : 1u), (uint64_t)N, nbatch};
    const uint64_t strides[3] = {sp.quad ? 128u : 32u, sl_bytes, sb_bytes};
    const uint32_t box[4] = {sp.quad ? 64u : 16u, 1, (uint32_t)kSTile, 1};
    if (!tma_encode_bf16(&kmap, k16_cache.ptr, 4, dims, strides, box, sp.quad ? 128 : 32))
      return RTP_ERR_CUDA;
    const size_t smem = score_smem_bytes(hm.G, sp.kw);
    // the whole carveout as shared memory: two CTAs per SM for kw <= 8
    if (cudaFuncSetAttribute(dec_score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess ||
        cudaFuncSetAttribute(dec_score_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared) != cudaSuccess)
      return RTP_ERR_CUDA;
    // CTAs per SM: two by the launch bounds, fewer if shared memory says so (the
    // occupancy query counts a TMEM-allocating kernel as one per SM; two CTAs
    // hold 2 x 128 of the 512 TMEM columns)
    int dev = 0, n_sm = 0, smem_sm = 0, smem_res = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) !=
            cudaSuccess ||
        cudaDeviceGetAttribute(&smem_res, cudaDevAttrReservedSharedMemoryPerBlock, dev) !=
            cudaSuccess)
      return RTP_ERR_CUDA;
    const int per_sm = std::max(1, std::min(2, smem_sm / ((int)smem + smem_res)));
    const int grid = std::max(1, std::min(sp.n_items, per_sm * n_sm));
    TraceScope tr("dec_score", s);
    dec_score_kernel<<<grid, kSThreads, smem, s>>>(kmap, sp);
    if ((st = check_cuda(cudaGetLastError())) != RTP_OK) return st;
  }
  return RTP_OK;
}
}  // namespace rtp

extern "C" rtp_status rtp_sparse_attn_decode_select(
    const rtp_shape* shape, const uint8_t* kv_role, int32_t k16_per_kv_head, rtp_view q,
    rtp_view k_cache, rtp_view v_cache, rtp_view q16, rtp_view k16_cache, rtp_select select,
    float p, int32_t top_k, float softmax_scale, rtp_view o, float* lse, float* thr,
    int32_t* jtie, int32_t* count, float* mass, uint32_t* block_mask, float* scores_out,
    void* ws, size_t ws_bytes, rtp_stream_t stream) {
  rtp_status st = check_shape(shape);
  if (st != RTP_OK) return st;
  if (shape->Lq != 1) return RTP_ERR_INVALID_ARG;
  if ((st = check_causal(shape)) != RTP_OK) return st;
  HeadMap hm;
  if ((st = make_headmap(shape, kv_role, k16_per_kv_head, &hm)) != RTP_OK) return st;
  if (select != RTP_SELECT_TOPP && select != RTP_SELECT_BLOCK_TOPP && select != RTP_SELECT_TOPK)
    return RTP_ERR_INVALID_ARG;
  if (select != RTP_SELECT_TOPK && !(p >= 0.f && p <= 1.f)) return RTP_ERR_INVALID_ARG;
  if (select == RTP_SELECT_TOPK && top_k < 1) return RTP_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f) || !isfinite(softmax_scale)) return RTP_ERR_INVALID_ARG;
  if (hm.G > 16 || (256 % hm.G) != 0) return RTP_ERR_UNSUPPORTED;
  if (shape->Lk > kMaxKeys) return RTP_ERR_UNSUPPORTED;
  const bool work = shape->B > 0 && hm.n_ret > 0;
  if (!work) return RTP_OK;
  if ((st = check_view(q, shape->H, kD, true)) != RTP_OK) return st;
  if ((st = check_view(k_cache, shape->Hkv, kD, true)) != RTP_OK) return st;
  if ((st = check_view(v_cache, shape->Hkv, kD, true)) != RTP_OK) return st;
  if ((st = check_view(o, shape->H, kD, true)) != RTP_OK) return st;
  if ((st = check_view(q16, hm.n_ret, kR, true)) != RTP_OK) return st;
  if ((st = check_view(k16_cache, hm.H_k16, kR, true)) != RTP_OK) return st;
  const DecodeWs L = decode_ws_layout(shape, hm);
  if (ws == nullptr || ws_bytes < L.total) return RTP_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  const int N = (int)(shape->q_pos0 + 1);  // keys 0..P
  const int nc = (N + kDecChunk - 1) / kDecChunk;
  const int groups = shape->B * hm.n_rkv;
  auto at = [&](size_t off) { return static_cast<void*>(w + off); };

  if ((st = decode_score_pass(shape, hm, k16_per_kv_head, q16, k16_cache, ws, L, s,
                              select == RTP_SELECT_BLOCK_TOPP)) != RTP_OK)
    return st;
  if (scores_out != nullptr && L.rows > 0 &&
      cudaMemcpy2DAsync(scores_out, (size_t)N * 4, at(L.scores), (size_t)L.Lk_pad * 4,
                        (size_t)N * 4, (size_t)L.rows, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return RTP_ERR_CUDA;
  if (select != RTP_SELECT_TOPP) {  // static top-k or block-level top-p (decode_variants.cu)
    DecodeLists dl;
    if ((st = decode_variant_select(shape, hm, select, p, top_k, ws, L, thr, jtie, count, mass,
                                    block_mask, &dl, s)) != RTP_OK)
      return st;
    return decode_list_attention(shape, hm, q, k_cache, v_cache, softmax_scale, o, lse, dl, s);
  }
  {  // 2. per-row merge
    MergeParams mp;
    mp.hist_m = static_cast<const unsigned long long*>(at(L.hist_m));
    mp.hist_c = static_cast<const uint32_t*>(at(L.hist_c));
    mp.flags = static_cast<const uint32_t*>(at(L.flags));
    mp.rowsel = static_cast<RowSel*>(at(L.rowsel));
    mp.p = p;
    TraceScope tr("dec_merge", s);
    if ((st = check_cuda(launch_dependent(dec_merge_kernel, dim3(L.rows), dim3(kThreads), 0, s,
                                          mp))) != RTP_OK)
      return st;
  }
  {  // 3. collect, compact, exact cut
    CollectParams cp;
    cp.scores = static_cast<const float*>(at(L.scores));
    cp.rowsel = static_cast<const RowSel*>(at(L.rowsel));
    cp.sub_m = static_cast<unsigned long long*>(at(L.sub_m));
    cp.sub_c = static_cast<uint32_t*>(at(L.sub_c));
    cp.cand = static_cast<unsigned long long*>(at(L.cand));
    cp.ncand = static_cast<uint32_t*>(at(L.ncand));
    cp.list = static_cast<uint2*>(at(L.list));
    cp.lcount = static_cast<int32_t*>(at(L.lcount));
    cp.loff = static_cast<int32_t*>(at(L.loff));
    cp.counter = static_cast<uint32_t*>(at(L.counter));
    cp.rowres = static_cast<RowRes*>(at(L.rowres));
    cp.thr = thr;
    cp.jtie = jtie;
    cp.count = count;
    cp.mass = mass;
    cp.status = static_cast<DevStatus*>(ws);
    cp.N = N;
    cp.Lk_pad = L.Lk_pad;
    cp.nc = nc;
    cp.n_ret = hm.n_ret;
    cp.n_rkv = hm.n_rkv;
    cp.G = hm.G;
    cp.p = p;
    const size_t smem = sizeof(CollectSmem);
    if (cudaFuncSetAttribute(dec_collect_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return RTP_ERR_CUDA;
    {
      TraceScope tr("dec_collect", s);
      if ((st = check_cuda(launch_dependent(dec_collect_kernel, dim3(nc, groups), dim3(kThreads),
                                            smem, s, cp))) != RTP_OK)
        return st;
    }
    const size_t rsmem = sizeof(ResolveSmem);
    if (cudaFuncSetAttribute(dec_resolve_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)rsmem) != cudaSuccess)
      return RTP_ERR_CUDA;
    TraceScope tr("dec_resolve", s);
    if ((st = check_cuda(launch_dependent(dec_resolve_kernel, dim3(L.rows), dim3(kThreads), rsmem,
                                          s, cp))) != RTP_OK)
      return st;
  }
  // 4. attention over the kept union
  DecodeLists dl;
  dl.list = static_cast<const uint2*>(at(L.list));
  dl.lcount = static_cast<const int32_t*>(at(L.lcount));
  dl.scores = static_cast<const float*>(at(L.scores));
  dl.rowres = static_cast<const RowRes*>(at(L.rowres));
  dl.part = static_cast<float*>(at(L.part));
  dl.Lk_pad = L.Lk_pad;
  dl.n_chunks = nc;
  dl.n_splits = decode_list_splits(groups, nc);
  if (dl.n_splits > L.n_splits) return RTP_ERR_WORKSPACE_TOO_SMALL;
  return decode_list_attention(shape, hm, q, k_cache, v_cache, softmax_scale, o, lse, dl, s);
}

extern "C" rtp_status rtp_sparse_attn_decode(const rtp_shape* shape, const uint8_t* kv_role,
                                             int32_t k16_per_kv_head, rtp_view q,
                                             rtp_view k_cache, rtp_view v_cache, rtp_view q16,
                                             rtp_view k16_cache, float p, float softmax_scale,
                                             rtp_view o, float* lse, float* thr, int32_t* jtie,
                                             int32_t* count, float* mass, void* ws,
                                             size_t ws_bytes, rtp_stream_t stream) {
  return rtp_sparse_attn_decode_select(shape, kv_role, k16_per_kv_head, q, k_cache, v_cache, q16,
                                       k16_cache, RTP_SELECT_TOPP, p, 0, softmax_scale, o, lse,
                                       thr, jtie, count, mass, nullptr, nullptr, ws, ws_bytes,
                                       stream);
}
