// decode_variants.cu -- the two other token-selection rules of a retrieval
// decode step, over the indexer scores the score pass of decode_select.cu left
// in the workspace ([rows][Lk_pad] fp32, one row per (batch entry, retrieval
// query head)):
//
//   static top-k  the method's fixed-budget variant (section "Experimental
//                 Analysis" of the paper-graph-ui summary of arXiv 2605.16928,
//                 k = 4096 there): the k highest scores, ties to the lower
//                 index.  One CTA per row finds the k-th largest composite key
//                 (order-preserving score bits, then the complemented index) by
//                 11-bit radix digits over the stored scores until at most 4096
//                 keys share the prefix, then sorts those in shared memory.
//                 Counts are integers, so the cut is exact.
//   block top-p   the summary's sort-free decode selection ("Hardware-Aware
//                 Fast Top-p Decoding Kernel", steps 1-5): the score pass reduces
//                 64-key blocks to (max m_b, log-sum-exp l_b) as it scores them
//                 (fused, as the summary's kernel is); here a 256-bin histogram
//                 over [min m_b, max m_b] whose bins sum exp(l_b - max) as 2^-40
//                 fixed point (order-free, so deterministic), a walk down the
//                 bins to mass p, one bit per selected block.  One CTA per row.
//
// A list kernel then writes, per (batch entry, retrieval kv head) and chunk of
// 1024 keys, the ordered list of keys some head keeps with their kept-head bits,
// which the split-KV list attention of decode.cu consumes unchanged.
#include <algorithm>

#include "dec_bins.cuh"
#include "rtp_host.h"

namespace rtp {
namespace {

constexpr int kVThreads = 1024;
constexpr int kVCap = 4096;                      // keys one CTA sorts at the end
constexpr int kVIdxBits = 21;
constexpr unsigned long long kVIdxMask = (1ull << kVIdxBits) - 1;
constexpr int kVKeyBits = 32 + kVIdxBits;        // 53-bit composite keys
constexpr int kVDigit = 11;                      // radix digit width
constexpr int kVBuckets = 1 << kVDigit;

struct VarParams {
  const float* scores;      // [rows][Lk_pad]
  const uint32_t* hist_c;   // [rows][kDecGBins]: keys per absolute score bin
  const uint32_t* flags;    // [rows]: 1 = a score fell outside the histogram's range
  RowRes* rowres;           // [rows]
  float2* blk;              // [rows][n_blk]: (m_b, l_b)
  uint32_t* bmask;          // [rows][n_bwords]
  uint32_t* bmask_out;      // caller's [rows][out_words] or null
  float* thr;
  int32_t* jtie;
  int32_t* count;
  float* mass;
  DevStatus* status;
  int N, Lk_pad, n_blk, n_bwords, out_words, top_k;
  float p;
};

__device__ __forceinline__ unsigned long long vkey(float s, int j) {
  return ((unsigned long long)score_key(s) << kVIdxBits) | (kVIdxMask - (unsigned long long)j);
}
__device__ __forceinline__ float vkey_score(unsigned long long ck) {
  const uint32_t key = (uint32_t)(ck >> kVIdxBits);
  const uint32_t b = (key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key;
  return __uint_as_float(b);
}
__device__ __forceinline__ float vexp(float x) {  // e^x, x <= 0: the reported mass only
  return exp2f(x * kLog2e);
}

__device__ float block_max_f(float v, float* red) {
  v = warp_max(v);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float m = -INFINITY;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, red[w]);
  __syncthreads();
  return m;
}

__device__ float block_min_f(float v, float* red) {
  return -block_max_f(-v, red);
}

__device__ unsigned long long block_sum_ull(unsigned long long v, unsigned long long* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  unsigned long long s = 0;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) s += red[w];
  __syncthreads();
  return s;
}

// Bitonic sort of a[0..n) descending (zero padding to a power of two), one block.
__device__ void vsort_desc(unsigned long long* a, int n) {
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

// ------------------------------------------------------------------ static top-k
struct TopkSmem {
  unsigned long long cand[kVCap];
  uint32_t hc[kVBuckets];
  unsigned long long hm[kVBuckets];
  unsigned long long ured[32];
  float fred[32];
  uint32_t wc[32];
  unsigned long long wm[32];
  int ncand;
  int s_d;
  uint32_t s_cnt, s_nin;
  unsigned long long s_acc;
};

__global__ void __launch_bounds__(kVThreads) dec_topk_kernel(const VarParams p) {
  griddep_wait();  // launched as a dependent of the score pass
  extern __shared__ __align__(16) unsigned char smem_raw[];
  TopkSmem& sm = *reinterpret_cast<TopkSmem*>(smem_raw);
  const int row = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int N = p.N;
  const float* srow = p.scores + (int64_t)row * p.Lk_pad;
  RowRes rr;
  if (p.top_k >= N) {  // every key
    rr.t = -INFINITY;
    rr.jtie = N - 1;
    rr.count = N;
    rr.mass = 1.f;
  } else {
    // Pick the first digit level: the score pass's absolute bins when every
    // score fell inside them (one more pass then collects the crossing bin),
    // else 11-bit radix digits of the composite keys.
    const bool use_hist = p.flags[row] == 0u;
    float m;  // mass reference >= every score: the top occupied bin's upper edge, or the max
    int pb = 0, gstar = 0;  // the crossing absolute bin (use_hist)
    unsigned long long prefix = 0, acc_above = 0, Z = 0;
    uint32_t need = (uint32_t)p.top_k, n_in = (uint32_t)N;
    // inclusive scan over 2048 buckets in descending order (thread t: positions
    // 2t, 2t + 1); returns the crossing position's bucket via shared memory
    auto cross = [&](const uint32_t* hc, const unsigned long long* hm, int nbk) {
      uint32_t c2[2] = {0, 0};
      unsigned long long m2[2] = {0, 0};
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int pos = 2 * tid + u;
        if (pos < nbk) {
          c2[u] = hc[nbk - 1 - pos];
          m2[u] = hm ? hm[nbk - 1 - pos] : 0ull;
        }
      }
      uint32_t ci = c2[0] + c2[1];
      unsigned long long mi = m2[0] + m2[1];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t cy = __shfl_up_sync(0xffffffffu, ci, o);
        const unsigned long long my = __shfl_up_sync(0xffffffffu, mi, o);
        if (lane >= o) {
          ci += cy;
          mi += my;
        }
      }
      if (lane == 31) {
        sm.wc[warp] = ci;
        sm.wm[warp] = mi;
      }
      __syncthreads();
      uint32_t cb = ci - c2[0] - c2[1];
      unsigned long long mb = mi - m2[0] - m2[1];
      for (int w2 = 0; w2 < warp; ++w2) {
        cb += sm.wc[w2];
        mb += sm.wm[w2];
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int pos = 2 * tid + u;
        if (pos < nbk && c2[u] > 0 && cb < need && cb + c2[u] >= need) {
          sm.s_d = nbk - 1 - pos;  // one bucket crosses: need is within it
          sm.s_cnt = cb;
          sm.s_acc = mb;
          sm.s_nin = c2[u];
        }
        cb += c2[u];
        mb += m2[u];
      }
      __syncthreads();
    };
    if (use_hist) {
      const uint32_t* hrow = p.hist_c + (int64_t)row * kDecGBins;
      int top = -1;
      for (int g = tid; g < kDecGBins; g += kVThreads)
        if (hrow[g]) top = max(top, g);
      top = (int)block_max_f((float)top, sm.fred);
      m = (float)(top + kDecGLo + 1) / kDecKappa;
      cross(hrow, nullptr, kDecGBins);
      gstar = sm.s_d + kDecGLo;  // the crossing absolute bin
      need -= sm.s_cnt;
      n_in = sm.s_nin;
      // one pass: Z, the mass above the crossing bin, its keys as candidates
      if (tid == 0) sm.ncand = 0;
      __syncthreads();
      unsigned long long zl = 0, al = 0;
      for (int j = tid; j < N; j += kVThreads) {
        const float s = srow[j];
        const unsigned long long w = mass_fixed40(vexp(s - m));
        const int bb = sbin(s);
        zl += w;
        if (bb > gstar) {
          al += w;
        } else if (bb == gstar && n_in <= (uint32_t)kVCap) {
          const int idx = atomicAdd(&sm.ncand, 1);
          if (idx < kVCap) sm.cand[idx] = vkey(s, j);
        }
      }
      Z = block_sum_ull(zl, sm.ured);
      acc_above = block_sum_ull(al, sm.ured);
      if (n_in > (uint32_t)kVCap) {  // a crowded bin: radix digits below its bin bits
        prefix = 0;
        pb = 0;
      }
    } else {
      float mx = -INFINITY;
      for (int j = tid; j < N; j += kVThreads) mx = fmaxf(mx, srow[j]);
      m = block_max_f(mx, sm.fred);
      unsigned long long zl = 0;
      for (int j = tid; j < N; j += kVThreads) zl += mass_fixed40(vexp(srow[j] - m));
      Z = block_sum_ull(zl, sm.ured);
    }
    // radix levels over the composite keys (restricted to the crossing bin when
    // the histogram chose one) while too many keys share the prefix
    const bool radix = !use_hist || n_in > (uint32_t)kVCap;
    while (radix && n_in > (uint32_t)kVCap && pb < kVKeyBits) {
      const int w = min(kVDigit, kVKeyBits - pb);
      const int nbk = 1 << w;
      for (int d = tid; d < nbk; d += kVThreads) {
        sm.hc[d] = 0;
        sm.hm[d] = 0;
      }
      __syncthreads();
      for (int j = tid; j < N; j += kVThreads) {
        const float s = srow[j];
        if (use_hist && sbin(s) != gstar) continue;
        const unsigned long long ck = vkey(s, j);
        if (pb > 0 && (ck >> (kVKeyBits - pb)) != prefix) continue;
        const int d = (int)((ck >> (kVKeyBits - pb - w)) & (unsigned long long)(nbk - 1));
        atomicAdd(&sm.hc[d], 1u);
        atomicAdd(&sm.hm[d], mass_fixed40(vexp(s - m)));
      }
      __syncthreads();
      cross(sm.hc, sm.hm, nbk);
      need -= sm.s_cnt;
      acc_above += sm.s_acc;
      n_in = sm.s_nin;
      prefix = (prefix << w) | (unsigned long long)sm.s_d;
      pb += w;
      __syncthreads();
    }
    if (radix) {  // the keys sharing the prefix
      if (tid == 0) sm.ncand = 0;
      __syncthreads();
      for (int j = tid; j < N; j += kVThreads) {
        const float s = srow[j];
        if (use_hist && sbin(s) != gstar) continue;
        const unsigned long long ck = vkey(s, j);
        if (pb > 0 && (ck >> (kVKeyBits - pb)) != prefix) continue;
        const int idx = atomicAdd(&sm.ncand, 1);
        if (idx < kVCap) sm.cand[idx] = ck;
      }
    }
    __syncthreads();
    // sorted, the cut is the need-th of them
    const int n = min(sm.ncand, kVCap);
    if (sm.ncand > kVCap && tid == 0) set_status(p.status, RTP_ERR_DEVICE_TIMEOUT, 41);
    vsort_desc(sm.cand, n);
    const int cut = min((int)need, n) - 1;
    unsigned long long part = 0;
    for (int a = tid; a <= cut; a += kVThreads) part += mass_fixed40(vexp(vkey_score(sm.cand[a]) - m));
    const unsigned long long kept = acc_above + block_sum_ull(part, sm.ured);
    const unsigned long long ck = sm.cand[max(cut, 0)];
    rr.t = vkey_score(ck);
    rr.jtie = (int32_t)(kVIdxMask - (ck & kVIdxMask));
    rr.count = p.top_k;
    rr.mass = Z > 0 ? (float)((double)kept / (double)Z) : 1.f;
  }
  if (tid == 0) {
    p.rowres[row] = rr;
    if (p.thr) p.thr[row] = rr.t;
    if (p.jtie) p.jtie[row] = rr.jtie;
    if (p.count) p.count[row] = rr.count;
    if (p.mass) p.mass[row] = rr.mass;
  }
}

// ------------------------------------------------------------------ block top-p
struct BlockSmem {
  unsigned long long hist[kDecHBins];
  unsigned long long ured[32];
  float fred[32];
  int s_kstar;
  unsigned long long s_kept, s_total;
};

// bin = min(255, floor(((m - lo) / (hi - lo)) * 256)) in fp64; 255 when hi == lo.
__device__ __forceinline__ int hbin(float m, float lo, float hi) {
  if (!(hi > lo)) return kDecHBins - 1;
  const double x = floor((((double)m - (double)lo) / ((double)hi - (double)lo)) * (double)kDecHBins);
  return x < (double)(kDecHBins - 1) ? (int)x : kDecHBins - 1;
}

__device__ __forceinline__ unsigned long long bmass_fixed(float l, float hi) {
  // exp(l_b - hi) <= 64 for a 64-key block; 2^-40 units (< 2^47 each)
  return (unsigned long long)__double2ull_rz(exp((double)l - (double)hi) * kFixedOne);
}

__global__ void __launch_bounds__(kVThreads) dec_block_topp_kernel(const VarParams p) {
  griddep_wait();  // launched as a dependent of the score pass
  __shared__ BlockSmem sm;
  const int row = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int N = p.N;
  const int nb = (N + kDecBlk - 1) / kDecBlk;
  float2* brow = p.blk + (int64_t)row * p.n_blk;
  // 1-2. per block: max and log-sum-exp, written by the score pass
  float lo = INFINITY, hi = -INFINITY;
  for (int bb = tid; bb < nb; bb += kVThreads) {
    const float mb = brow[bb].x;
    lo = fminf(lo, mb);
    hi = fmaxf(hi, mb);
  }
  for (int k = tid; k < kDecHBins; k += kVThreads) sm.hist[k] = 0;
  lo = block_min_f(lo, sm.fred);
  hi = block_max_f(hi, sm.fred);
  // 3. histogram over the block maxima
  for (int bb = tid; bb < nb; bb += kVThreads) {
    const float2 ml = brow[bb];
    atomicAdd(&sm.hist[hbin(ml.x, lo, hi)], bmass_fixed(ml.y, hi));
  }
  __syncthreads();
  // 4. walk the bins from the top (warp 0: lane owns bins 255 - 8 lane ... - 7)
  if (warp == 0) {
    unsigned long long hv[8], own = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      hv[i] = sm.hist[kDecHBins - 1 - (lane * 8 + i)];
      own += hv[i];
    }
    unsigned long long incl = own;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const unsigned long long total = __shfl_sync(0xffffffffu, incl, 31);
    const double T = (double)p.p * (double)total;
    unsigned long long cum = incl - own;
    int my = 0x7FFFFFFF;
    unsigned long long mycum = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (hv[i] == 0) continue;
      cum += hv[i];
      if (my == 0x7FFFFFFF && (double)cum >= T) {
        my = lane * 8 + i;
        mycum = cum;
      }
    }
    int pos = my;
    if (p.p >= 1.f) {  // every block, whatever the masses round to
      if (lane == 0) {
        sm.s_kstar = 0;
        sm.s_kept = total;
        sm.s_total = total;
      }
    } else {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) pos = min(pos, __shfl_xor_sync(0xffffffffu, pos, o));
      if (pos == 0x7FFFFFFF) {  // rounding kept T out of reach: every block
        if (lane == 0) {
          sm.s_kstar = 0;
          sm.s_kept = total;
          sm.s_total = total;
        }
      } else if (my == pos) {
        sm.s_kstar = kDecHBins - 1 - pos;
        sm.s_kept = mycum;
        sm.s_total = total;
      }
    }
  }
  __syncthreads();
  const int kstar = sm.s_kstar;
  // 5. one bit per block, and the kept key count
  uint32_t* mrow = p.bmask + (int64_t)row * p.n_bwords;
  uint32_t* orow = p.bmask_out ? p.bmask_out + (int64_t)row * p.out_words : nullptr;
  unsigned long long kept_keys = 0;
  const int nb32 = (nb + 31) / 32 * 32;
  for (int bb = tid; bb < nb32; bb += kVThreads) {
    bool on = false;
    if (bb < nb) {
      const float2 ml = brow[bb];
      on = hbin(ml.x, lo, hi) >= kstar;
      if (on) kept_keys += (unsigned long long)min(kDecBlk, N - bb * kDecBlk);
    }
    const uint32_t word = __ballot_sync(0xffffffffu, on);
    if (lane == 0) {
      mrow[bb >> 5] = word;
      if (orow) orow[bb >> 5] = word;
    }
  }
  const unsigned long long cnt = block_sum_ull(kept_keys, sm.ured);
  if (tid == 0) {
    RowRes rr;
    rr.t = -INFINITY;  // the attention reads kept bits only
    rr.jtie = N - 1;
    rr.count = (int32_t)cnt;
    rr.mass = sm.s_total > 0 ? (float)((double)sm.s_kept / (double)sm.s_total) : 1.f;
    p.rowres[row] = rr;
    if (p.count) p.count[row] = rr.count;
    if (p.mass) p.mass[row] = rr.mass;
  }
}

// ------------------------------------------------------------------ union lists
struct VListParams {
  const float* scores;
  const RowRes* rowres;
  const uint32_t* bmask;
  uint2* list;       // [groups][Lk_pad]
  int32_t* lcount;   // [groups][nc]
  int N, Lk_pad, nc, n_ret, n_rkv, G, n_bwords, block_mode;
};

constexpr int kLThreads = kDecChunk / 4;  // four keys per thread

__global__ void __launch_bounds__(kLThreads) dec_varlist_kernel(const VListParams p) {
  griddep_wait();  // launched as a dependent of the selection kernel
  __shared__ int wsum[kLThreads / 32];
  __shared__ RowRes rs[16];
  const int chunk = blockIdx.x, grp = blockIdx.y;
  const int b = grp / p.n_rkv, rk = grp % p.n_rkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = p.G;
  const int row0 = b * p.n_ret + rk * G;
  if (tid < G) rs[tid] = p.rowres[row0 + tid];
  __syncthreads();
  const int j0 = chunk * kDecChunk + tid * 4;
  uint32_t keep[4] = {0, 0, 0, 0};
  for (int h = 0; h < G; ++h) {
    if (p.block_mode) {
      const uint32_t word = p.bmask[(int64_t)(row0 + h) * p.n_bwords + (j0 >> 11)];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = j0 + e;
        if (j < p.N && ((word >> ((j >> 6) & 31)) & 1u)) keep[e] |= 1u << h;
      }
    } else {
      const float4 v =
          *reinterpret_cast<const float4*>(p.scores + (int64_t)(row0 + h) * p.Lk_pad + j0);
      const float vs[4] = {v.x, v.y, v.z, v.w};
      const float t = rs[h].t;
      const int jt = rs[h].jtie;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = j0 + e;
        if (j < p.N && (vs[e] > t || (vs[e] == t && j <= jt))) keep[e] |= 1u << h;
      }
    }
  }
  int cnt = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e) cnt += keep[e] != 0;
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  int off = incl - cnt;
  for (int w = 0; w < warp; ++w) off += wsum[w];
  uint2* dst = p.list + (int64_t)grp * p.Lk_pad + chunk * kDecChunk;
#pragma unroll
  for (int e = 0; e < 4; ++e)
    if (keep[e]) dst[off++] = make_uint2((uint32_t)(j0 + e), keep[e]);
  if (tid == kLThreads - 1) {
    int tot = 0;
    for (int w = 0; w < kLThreads / 32; ++w) tot += wsum[w];
    p.lcount[(int64_t)grp * p.nc + chunk] = tot;
  }
}

}  // namespace

rtp_status decode_variant_select(const rtp_shape* shape, const HeadMap& hm, rtp_select select,
                                 float p, int top_k, void* ws, const DecodeWs& L, float* thr,
                                 int32_t* jtie, int32_t* count, float* mass,
                                 uint32_t* block_mask, DecodeLists* lists, cudaStream_t s) {
  char* w = static_cast<char*>(ws);
  auto at = [&](size_t off) { return static_cast<void*>(w + off); };
  const int N = (int)(shape->q_pos0 + 1);
  const int nc = (N + kDecChunk - 1) / kDecChunk;
  const int groups = shape->B * hm.n_rkv;
  VarParams vp;
  memset(&vp, 0, sizeof(vp));
  vp.scores = static_cast<const float*>(at(L.scores));
  vp.hist_c = static_cast<const uint32_t*>(at(L.hist_c));
  vp.flags = static_cast<const uint32_t*>(at(L.flags));
  vp.rowres = static_cast<RowRes*>(at(L.rowres));
  vp.blk = static_cast<float2*>(at(L.blk));
  vp.bmask = static_cast<uint32_t*>(at(L.bmask));
  vp.bmask_out = block_mask;
  vp.thr = thr;
  vp.jtie = jtie;
  vp.count = count;
  vp.mass = mass;
  vp.status = static_cast<DevStatus*>(ws);
  vp.N = N;
  vp.Lk_pad = L.Lk_pad;
  vp.n_blk = L.n_blk;
  vp.n_bwords = L.n_bwords;
  vp.out_words = ((N + kDecBlk - 1) / kDecBlk + 31) / 32;
  vp.top_k = top_k;
  vp.p = p;
  rtp_status st;
  if (select == RTP_SELECT_TOPK) {
    const size_t smem = sizeof(TopkSmem);
    if (cudaFuncSetAttribute(dec_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return RTP_ERR_CUDA;
    TraceScope tr("dec_topk", s);
    if ((st = check_cuda(launch_dependent(dec_topk_kernel, dim3(L.rows), dim3(kVThreads), smem, s,
                                          vp))) != RTP_OK)
      return st;
  } else {
    TraceScope tr("dec_block_topp", s);
    if ((st = check_cuda(launch_dependent(dec_block_topp_kernel, dim3(L.rows), dim3(kVThreads), 0,
                                          s, vp))) != RTP_OK)
      return st;
  }
  VListParams lp;
  lp.scores = vp.scores;
  lp.rowres = vp.rowres;
  lp.bmask = vp.bmask;
  lp.list = static_cast<uint2*>(at(L.list));
  lp.lcount = static_cast<int32_t*>(at(L.lcount));
  lp.N = N;
  lp.Lk_pad = L.Lk_pad;
  lp.nc = nc;
  lp.n_ret = hm.n_ret;
  lp.n_rkv = hm.n_rkv;
  lp.G = hm.G;
  lp.n_bwords = L.n_bwords;
  lp.block_mode = select == RTP_SELECT_BLOCK_TOPP ? 1 : 0;
  {
    TraceScope tr("dec_varlist", s);
    if ((st = check_cuda(launch_dependent(dec_varlist_kernel, dim3(nc, groups), dim3(kLThreads), 0,
                                          s, lp))) != RTP_OK)
      return st;
  }
  lists->list = lp.list;
  lists->lcount = lp.lcount;
  lists->scores = vp.scores;
  lists->rowres = vp.rowres;
  lists->part = static_cast<float*>(at(L.part));
  lists->Lk_pad = L.Lk_pad;
  lists->n_chunks = nc;
  lists->n_splits = decode_list_splits(groups, nc);
  if (lists->n_splits > L.n_splits) return RTP_ERR_WORKSPACE_TOO_SMALL;
  return RTP_OK;
}

}  // namespace rtp
