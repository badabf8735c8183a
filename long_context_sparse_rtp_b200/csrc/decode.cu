// decode.cu -- single-token decode: retrieval heads (rtp_sparse_attn_decode) and
// the range-mode decode attention used by local and dense heads.
//
// Retrieval decode for one query token per batch entry ("Dynamic Top-p
// Selection Mechanism" and the decode flow of the paper-graph-ui summary of
// arXiv 2605.16928), per kv group of G query heads:
//   1. score     stream the k16 cache once (HBM-bound), s = q16 . k16 in fp32,
//                scores kept in the workspace (L2-resident), chunk maxima;
//   2. histogram Z and a 256-bin mass histogram above c0 = m - ln(N/(1-p)) - 1,
//                40-bit fixed-point sums (exact, order-free); the last CTA of a
//                row (arrival counter) finds the crossing bin, collects the keys
//                in it, sorts them and walks to the exact cut (t, jtie);
//   3. compact   one ordered list per kv group of the union of kept keys with a
//                per-head bit mask (the kv-level "memory sparsity" set);
//   4. attend    split-KV over the list: gathered K/V rows staged in shared
//                memory with 16-byte cp.async, tensor-core QK^T / PV with the
//                G heads as mma rows, per-head masks, online softmax; the last
//                CTA of a group merges the splits.
#include <algorithm>
#include <mutex>

#include "rtp_host.h"

namespace rtp {

rtp_status prefill_local(const rtp_shape*, const HeadMap&, int, int, const rtp_view&,
                         const rtp_view&, const rtp_view&, float, const rtp_view&, float*,
                         cudaStream_t);
rtp_status prefill_dense(const rtp_shape*, const rtp_view&, const rtp_view&, const rtp_view&,
                         float, const rtp_view&, float*, cudaStream_t);
rtp_status prefill_sparse(const rtp_shape*, const HeadMap&, const rtp_view&, const rtp_view&,
                          const rtp_view&, const rtp_view&, const rtp_view&, const float*,
                          const int32_t*, float, const rtp_view&, float*, cudaStream_t);

namespace {

constexpr int kIdxBits = 21;
constexpr unsigned long long kIdxMask = (1ull << kIdxBits) - 1;
constexpr int kKeyBits = 32 + kIdxBits;

__device__ __forceinline__ float mass_w(float s, float m) {
  return exp2f(__fmul_rn(__fsub_rn(s, m), kLog2e));
}
__device__ __forceinline__ int dbin0(float s, float m, float scale) {
  const int b = (int)__fmul_rn(__fsub_rn(m, s), scale);
  return b < kDecBins - 1 ? b : kDecBins - 1;
}
__device__ __forceinline__ unsigned long long comp_key(float s, int j) {
  return ((unsigned long long)score_key(s) << kIdxBits) | (kIdxMask - (unsigned long long)j);
}
__device__ __forceinline__ float key_score(uint32_t key) {
  const uint32_t b = (key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key;
  return __uint_as_float(b);
}

// ------------------------------------------------------------------ 1. score
struct ScoreParams {
  const uint16_t* q16;
  int64_t q16_sb;
  const uint16_t* k16;
  int64_t k16_sb, k16_sl;
  float* scores;
  float* cmax;
  unsigned long long* hist_m;   // zeroed here for this group's rows
  uint32_t* hist_c;
  unsigned long long* zsum;
  uint32_t* counter;
  uint32_t* mcount;
  int N, Lk_pad, n_chunks, n_ret, n_rkv, G;
  int per_kv;
};

constexpr int kScoreThreads = 256;

__global__ void __launch_bounds__(kScoreThreads) dec_score_kernel(const ScoreParams p) {
  extern __shared__ __align__(16) float sc[];  // [G][kDecChunk + 4]
  const int chunk = blockIdx.x;
  const int grp = blockIdx.y;  // b * n_rkv + rk
  const int b = grp / p.n_rkv, rk = grp % p.n_rkv;
  const int tid = threadIdx.x;
  const int G = p.G;
  const int hh = tid % G;  // G divides 256: constant per thread
  const int hr = rk * G + hh;
  float q[kR];
  {
    const uint16_t* qp = p.q16 + b * p.q16_sb + (int64_t)hr * kR;
    const uint4 a = *reinterpret_cast<const uint4*>(qp);
    const uint4 c = *reinterpret_cast<const uint4*>(qp + 8);
    q[0] = bf16_lo(a.x); q[1] = bf16_hi(a.x); q[2] = bf16_lo(a.y); q[3] = bf16_hi(a.y);
    q[4] = bf16_lo(a.z); q[5] = bf16_hi(a.z); q[6] = bf16_lo(a.w); q[7] = bf16_hi(a.w);
    q[8] = bf16_lo(c.x); q[9] = bf16_hi(c.x); q[10] = bf16_lo(c.y); q[11] = bf16_hi(c.y);
    q[12] = bf16_lo(c.z); q[13] = bf16_hi(c.z); q[14] = bf16_lo(c.w); q[15] = bf16_hi(c.w);
  }
  if (chunk == 0) {
    // later kernels accumulate into these with atomics: start them at zero
    const int row0 = b * p.n_ret + rk * G;
    for (int x = tid; x < G * kDecBins; x += kScoreThreads) {
      p.hist_m[(int64_t)row0 * kDecBins + x] = 0ull;
      p.hist_c[(int64_t)row0 * kDecBins + x] = 0u;
    }
    if (tid < G) {
      p.zsum[row0 + tid] = 0ull;
      p.counter[row0 + tid] = 0u;
    }
    if (tid == 0) p.mcount[grp] = 0u;
  }
  const int slot = p.per_kv ? rk : hr;
  const uint16_t* kb = p.k16 + b * p.k16_sb + (int64_t)slot * kR;
  const int j0 = chunk * kDecChunk;
  const int pairs = kDecChunk * G;
  constexpr int kUnroll = 4;
  for (int base = 0; base < pairs; base += kScoreThreads * kUnroll) {
    uint4 ka[kUnroll], kc[kUnroll];
    int tok[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int pr = base + u * kScoreThreads + tid;
      tok[u] = pr / G;
      const int j = j0 + tok[u];
      if (pr < pairs && j < p.N) {
        const uint16_t* src = kb + (int64_t)j * p.k16_sl;
        ka[u] = __ldcs(reinterpret_cast<const uint4*>(src));
        kc[u] = __ldcs(reinterpret_cast<const uint4*>(src + 8));
      } else {
        ka[u] = make_uint4(0, 0, 0, 0);
        kc[u] = ka[u];
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int pr = base + u * kScoreThreads + tid;
      if (pr >= pairs) continue;
      const uint32_t w[8] = {ka[u].x, ka[u].y, ka[u].z, ka[u].w, kc[u].x, kc[u].y, kc[u].z, kc[u].w};
      float s = 0.f;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        s = fmaf(q[2 * c], bf16_lo(w[c]), s);
        s = fmaf(q[2 * c + 1], bf16_hi(w[c]), s);
      }
      s = s + 0.0f;
      const int j = j0 + tok[u];
      sc[hh * (kDecChunk + 4) + tok[u]] = (j < p.N) ? s : -INFINITY;
    }
  }
  __syncthreads();
  const int warp = tid >> 5, lane = tid & 31;
  for (int h = warp; h < G; h += kScoreThreads / 32) {
    const float* row = sc + h * (kDecChunk + 4);
    float mx = -INFINITY;
    float* dst = p.scores + ((int64_t)(b * p.n_ret + rk * G + h)) * p.Lk_pad + j0;
    for (int x = lane * 4; x < kDecChunk; x += 128) {
      const float4 v = *reinterpret_cast<const float4*>(row + x);
      mx = fmaxf(mx, fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w)));
      *reinterpret_cast<float4*>(dst + x) = v;
    }
    mx = warp_max(mx);
    if (lane == 0) p.cmax[(int64_t)(b * p.n_ret + rk * G + h) * p.n_chunks + chunk] = mx;
  }
}

// ------------------------------------------------------------------ 2. histogram + resolve
struct HistParams {
  const float* scores;
  const float* cmax;
  unsigned long long* hist_m;
  uint32_t* hist_c;
  unsigned long long* zsum;
  uint32_t* counter;
  RowRes* rowres;
  float* thr;
  int32_t* jtie;
  int32_t* count;
  float* mass;
  DevStatus* status;
  int N, Lk_pad, n_chunks, cmax_stride;
  float p;
};

constexpr int kHistThreads = 256;

struct HistSmem {
  unsigned long long hm[kDecBins];
  uint32_t hc[kDecBins];
  unsigned long long cand[kDecCap];
  unsigned long long red[kHistThreads / 32];
  unsigned long long tsum[kHistThreads];
  float fred[kHistThreads / 32];
  int ncand;
  int is_last;
  int cut;
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
  return s;
}

__device__ float block_max(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_max(v);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float m = -INFINITY;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, red[w]);
  return m;
}

// Bitonic sort of sm.cand[0..n) descending (n padded to a power of two with 0).
__device__ void sort_desc(unsigned long long* a, int n) {
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

__global__ void __launch_bounds__(kHistThreads) dec_hist_kernel(const HistParams p) {
  __shared__ HistSmem sm;
  const int row = blockIdx.y;
  const int tid = threadIdx.x;
  const float* srow = p.scores + (int64_t)row * p.Lk_pad;

  // row max from the chunk maxima
  float mx = -INFINITY;
  for (int c = tid; c < p.n_chunks; c += kHistThreads)
    mx = fmaxf(mx, p.cmax[(int64_t)row * p.cmax_stride + c]);
  const float m = block_max(mx, sm.fred);
  const float R = (float)(log((double)p.N / (1.0 - (double)p.p)) + 1.0);
  const float c0 = m - R;
  const float scale = (float)kDecBins / R;

  for (int b = tid; b < kDecBins; b += kHistThreads) {
    sm.hm[b] = 0;
    sm.hc[b] = 0;
  }
  __syncthreads();
  const int j0 = blockIdx.x * kDecHistChunk;
  const int j1 = min(p.N, j0 + kDecHistChunk);
  unsigned long long z = 0;
  for (int j = j0 + tid * 4; j < j1; j += kHistThreads * 4) {
    const float4 v4 = *reinterpret_cast<const float4*>(srow + j);
    const float vs[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (j + e >= j1) break;
      const float s = vs[e];
      const unsigned long long f = mass_fixed40(mass_w(s, m));
      z += f;
      if (s >= c0) {
        const int bin = dbin0(s, m, scale);
        atomicAdd(&sm.hm[bin], f);
        atomicAdd(&sm.hc[bin], 1u);
      }
    }
  }
  z = block_sum_u64(z, sm.red);
  if (tid == 0) atomicAdd(&p.zsum[row], z);
  for (int b = tid; b < kDecBins; b += kHistThreads) {
    if (sm.hc[b]) {
      atomicAdd(&p.hist_m[(int64_t)row * kDecBins + b], sm.hm[b]);
      atomicAdd(&p.hist_c[(int64_t)row * kDecBins + b], sm.hc[b]);
    }
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) sm.is_last = (atomicAdd(&p.counter[row], 1u) == gridDim.x - 1);
  __syncthreads();
  if (!sm.is_last) return;
  __threadfence();

  // ---------------- last CTA of this row: exact cut
  const unsigned long long Z = __ldcg(&p.zsum[row]);
  const double T = (double)p.p * (double)Z;
  for (int b = tid; b < kDecBins; b += kHistThreads) {
    sm.hm[b] = __ldcg(&p.hist_m[(int64_t)row * kDecBins + b]);
    sm.hc[b] = __ldcg(&p.hist_c[(int64_t)row * kDecBins + b]);
  }
  __syncthreads();
  // crossing bin (one thread; 256 bins)
  __shared__ unsigned long long s_acc;
  __shared__ uint32_t s_cnt, s_nin;
  __shared__ int s_k0;
  if (tid == 0) {
    unsigned long long acc = 0;
    uint32_t cnt = 0, nin = 0;
    int last = -1, k = -1;
    for (int b = 0; b < kDecBins; ++b) {
      if (sm.hc[b] == 0) continue;
      last = b;
      if ((double)(acc + sm.hm[b]) >= T) {
        k = b;
        nin = sm.hc[b];
        break;
      }
      acc += sm.hm[b];
      cnt += sm.hc[b];
    }
    if (k < 0) {
      k = last;
      acc -= sm.hm[last];
      cnt -= sm.hc[last];
      nin = sm.hc[last];
    }
    s_acc = acc;
    s_cnt = cnt;
    s_nin = nin;
    s_k0 = k;
  }
  __syncthreads();
  unsigned long long acc_above = s_acc;
  uint32_t cnt_above = s_cnt;
  uint32_t n_in = s_nin;
  const int k0 = s_k0;
  // radix refinement (8-bit digits) while the crossing bin is too full
  int pb = 0;
  unsigned long long prefix = 0;
  {
    const float hi_s = m - (float)k0 / scale, lo_s = m - (float)(k0 + 1) / scale;
    const float margin = 1e-5f * (fabsf(m) + R + 1.f);
    const unsigned long long kl = (unsigned long long)score_key(lo_s - margin) << kIdxBits;
    const unsigned long long kh =
        ((unsigned long long)score_key(hi_s + margin) << kIdxBits) | kIdxMask;
    pb = (kl == kh) ? kKeyBits : (__clzll(kl ^ kh) - (64 - kKeyBits));
    prefix = pb > 0 ? (kh >> (kKeyBits - pb)) : 0ull;
  }
  auto member = [&](float s, int j, unsigned long long& ck) -> bool {
    if (s < c0 || dbin0(s, m, scale) != k0) return false;
    ck = comp_key(s, j);
    return pb == 0 || (ck >> (kKeyBits - pb)) == prefix;
  };
  for (int lvl = 0; lvl < 8 && n_in > (uint32_t)kDecCap && pb < kKeyBits; ++lvl) {
    const int w = min(8, kKeyBits - pb);
    for (int b = tid; b < kDecBins; b += kHistThreads) {
      sm.hm[b] = 0;
      sm.hc[b] = 0;
    }
    __syncthreads();
    for (int j = tid; j < p.N; j += kHistThreads) {
      const float s = srow[j];
      unsigned long long ck;
      if (!member(s, j, ck)) continue;
      const int digit = (int)((ck >> (kKeyBits - pb - w)) & ((1ull << w) - 1));
      const int bin = (1 << w) - 1 - digit;
      atomicAdd(&sm.hm[bin], mass_fixed40(mass_w(s, m)));
      atomicAdd(&sm.hc[bin], 1u);
    }
    __syncthreads();
    if (tid == 0) {
      unsigned long long acc = acc_above;
      uint32_t cnt = cnt_above, nin = 0;
      int last = -1, k = -1;
      for (int b = 0; b < (1 << w); ++b) {
        if (sm.hc[b] == 0) continue;
        last = b;
        if ((double)(acc + sm.hm[b]) >= T) {
          k = b;
          nin = sm.hc[b];
          break;
        }
        acc += sm.hm[b];
        cnt += sm.hc[b];
      }
      if (k < 0) {
        k = last;
        acc -= sm.hm[last];
        cnt -= sm.hc[last];
        nin = sm.hc[last];
      }
      s_acc = acc;
      s_cnt = cnt;
      s_nin = nin;
      s_k0 = (1 << w) - 1 - k;  // digit
    }
    __syncthreads();
    acc_above = s_acc;
    cnt_above = s_cnt;
    n_in = s_nin;
    prefix = (prefix << w) | (unsigned long long)s_k0;
    pb += w;
    __syncthreads();
  }
  // collect the crossing keys
  if (tid == 0) sm.ncand = 0;
  __syncthreads();
  for (int j = tid; j < p.N; j += kHistThreads) {
    const float s = srow[j];
    unsigned long long ck;
    if (!member(s, j, ck)) continue;
    const int idx = atomicAdd(&sm.ncand, 1);
    if (idx < kDecCap) sm.cand[idx] = ck;
  }
  __syncthreads();
  int n = sm.ncand;
  if (n > kDecCap || n == 0) {
    if (tid == 0) set_status(p.status, RTP_ERR_DEVICE_TIMEOUT, 22);
    n = n == 0 ? 1 : kDecCap;
    if (sm.ncand == 0 && tid == 0) sm.cand[0] = comp_key(m, 0);
    __syncthreads();
  }
  sort_desc(sm.cand, n);
  // walk: per-thread contiguous segments, block scan of the segment sums
  const int per = (n + kHistThreads - 1) / kHistThreads;
  const int a0 = tid * per, a1 = min(n, a0 + per);
  unsigned long long seg = 0;
  for (int a = a0; a < a1; ++a)
    seg += mass_fixed40(mass_w(key_score((uint32_t)(sm.cand[a] >> kIdxBits)), m));
  sm.tsum[tid] = seg;
  if (tid == 0) sm.cut = 0x7FFFFFFF;
  __syncthreads();
  unsigned long long before = acc_above;
  for (int q = 0; q < tid; ++q) before += sm.tsum[q];
  {
    unsigned long long cum = before;
    for (int a = a0; a < a1; ++a) {
      cum += mass_fixed40(mass_w(key_score((uint32_t)(sm.cand[a] >> kIdxBits)), m));
      if ((double)cum >= T) {
        atomicMin(&sm.cut, a);
        break;
      }
    }
  }
  __syncthreads();
  int cut = sm.cut;
  if (cut == 0x7FFFFFFF) cut = n - 1;
  if (tid == 0) {
    unsigned long long cum = acc_above;
    for (int a = 0; a <= cut; ++a)
      cum += mass_fixed40(mass_w(key_score((uint32_t)(sm.cand[a] >> kIdxBits)), m));
    const unsigned long long ck = sm.cand[cut];
    RowRes rr;
    rr.t = key_score((uint32_t)(ck >> kIdxBits));
    rr.jtie = (int32_t)(kIdxMask - (ck & kIdxMask));
    rr.count = (int32_t)(cnt_above + cut + 1);
    rr.mass = (float)((double)cum / (double)Z);
    p.rowres[row] = rr;
    if (p.thr) p.thr[row] = rr.t;
    if (p.jtie) p.jtie[row] = rr.jtie;
    if (p.count) p.count[row] = rr.count;
    if (p.mass) p.mass[row] = rr.mass;
    p.zsum[row] = 0;
    p.counter[row] = 0;
  }
  for (int b = tid; b < kDecBins; b += kHistThreads) {
    p.hist_m[(int64_t)row * kDecBins + b] = 0;
    p.hist_c[(int64_t)row * kDecBins + b] = 0;
  }
}

// p >= 1: every key kept.
__global__ void dec_all_kernel(RowRes* rowres, int rows, int N, float* thr, int32_t* jtie,
                               int32_t* count, float* mass) {
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= rows) return;
  RowRes rr;
  rr.t = -INFINITY;
  rr.jtie = N - 1;
  rr.count = N;
  rr.mass = 1.f;
  rowres[r] = rr;
  if (thr) thr[r] = rr.t;
  if (jtie) jtie[r] = rr.jtie;
  if (count) count[r] = rr.count;
  if (mass) mass[r] = rr.mass;
}

// ------------------------------------------------------------------ 3. compact
struct CompactParams {
  const float* scores;
  const RowRes* rowres;
  uint2* list;        // [groups][Lk_pad]: {j, head mask}
  int32_t* lcount;    // [groups][n_chunks]
  int N, Lk_pad, n_chunks, n_ret, n_rkv, G;
};

constexpr int kCompactThreads = 256;

__global__ void __launch_bounds__(kCompactThreads) dec_compact_kernel(const CompactParams p) {
  __shared__ float st[16];
  __shared__ int sj[16];
  __shared__ int wsum[kCompactThreads / 32];
  const int chunk = blockIdx.x, grp = blockIdx.y;
  const int b = grp / p.n_rkv, rk = grp % p.n_rkv;
  const int tid = threadIdx.x;
  const int G = p.G;
  const int row0 = b * p.n_ret + rk * G;
  if (tid < G) {
    st[tid] = p.rowres[row0 + tid].t;
    sj[tid] = p.rowres[row0 + tid].jtie;
  }
  __syncthreads();
  const int j0 = chunk * kDecChunk + tid * 4;
  uint32_t mask[4] = {0, 0, 0, 0};
  for (int h = 0; h < G; ++h) {
    const float4 v = *reinterpret_cast<const float4*>(p.scores + (int64_t)(row0 + h) * p.Lk_pad + j0);
    const float vs[4] = {v.x, v.y, v.z, v.w};
    const float t = st[h];
    const int jt = sj[h];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int j = j0 + e;
      const bool keep = j < p.N && (vs[e] > t || (vs[e] == t && j <= jt));
      mask[e] |= (uint32_t)keep << h;
    }
  }
  int cnt = (mask[0] != 0) + (mask[1] != 0) + (mask[2] != 0) + (mask[3] != 0);
  // block exclusive scan (ordered by token)
  const int lane = tid & 31, warp = tid >> 5;
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
    if (mask[e]) dst[off++] = make_uint2((uint32_t)(j0 + e), mask[e]);
  if (tid == kCompactThreads - 1) {
    int tot = 0;
    for (int w = 0; w < kCompactThreads / 32; ++w) tot += wsum[w];
    p.lcount[(int64_t)grp * p.n_chunks + chunk] = tot;
  }
}

// ------------------------------------------------------------------ 4. attend
struct DecAttnParams {
  const uint16_t* q; int64_t q_sb;       // query row of each batch entry
  const uint16_t* k; int64_t k_sb, k_sl;
  const uint16_t* v; int64_t v_sb, v_sl;
  uint16_t* o; int64_t o_sb;
  float* lse; int64_t lse_sb;            // lse[b*lse_sb + h] (Lq == 1)
  float scale_log2;
  int G, groups, n_splits;
  // list mode
  const uint2* list; const int32_t* lcount; int Lk_pad, n_chunks, chunks_per_split;
  // range mode
  int64_t P; int n_sink_eff; int64_t win_lo; int64_t n_keys; int keys_per_split;
  float* part;                            // [B*groups][n_splits][16][2+128]
  uint32_t* mcount;                       // [B*groups]
  int16_t kvh[kMaxHeads];                 // group -> kv head
};

constexpr int kDecThreads = 128;
constexpr int kTile = 64;

struct DecSmem {
  uint16_t q[16][kD];
  uint16_t k[2][kTile][kD];
  uint16_t v[2][kTile][kD];
  uint32_t mask[2][kTile];
  float wm[4][16], wl[4][16];
  float wo[4][16][kD];
  int is_last;
};

__device__ __forceinline__ uint32_t dswz(const uint16_t (*base)[kD], int r, int chunk) {
  return smem_u32(&base[r][((chunk ^ (r & 7)) << 3)]);
}

template <bool LIST>
__global__ void __launch_bounds__(kDecThreads) dec_attn_kernel(const DecAttnParams p) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  DecSmem& sm = *reinterpret_cast<DecSmem*>(smem_raw);
  const int split = blockIdx.x;
  const int gg = blockIdx.y;               // b * groups + group
  const int b = gg / p.groups, grp = gg % p.groups;
  const int kvh = p.kvh[grp];
  const int G = p.G;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const uint32_t allmask = (G >= 32) ? 0xFFFFFFFFu : ((1u << G) - 1u);

  // query rows: heads kvh*G .. +G-1 (rows >= G are zero)
  for (int c = tid; c < 16 * 16; c += kDecThreads) {
    const int r = c >> 4, ch = c & 15;
    uint4 val = make_uint4(0, 0, 0, 0);
    if (r < G)
      val = *reinterpret_cast<const uint4*>(p.q + b * p.q_sb + (int64_t)(kvh * G + r) * kD + ch * 8);
    *reinterpret_cast<uint4*>(&sm.q[r][((ch ^ (r & 7)) << 3)]) = val;
  }

  // this split's slots
  int64_t e_begin = 0, e_end = 0;  // range mode: virtual key index range
  int c_begin = 0, c_end = 0;      // list mode: chunk range
  int n_entries = 0;
  if (LIST) {
    c_begin = split * p.chunks_per_split;
    c_end = min(p.n_chunks, c_begin + p.chunks_per_split);
    for (int c = c_begin; c < c_end; ++c) n_entries += p.lcount[(int64_t)gg * p.n_chunks + c];
  } else {
    e_begin = (int64_t)split * p.keys_per_split;
    e_end = min(p.n_keys, e_begin + p.keys_per_split);
    n_entries = (int)max((int64_t)0, e_end - e_begin);
  }
  const int n_tiles = (n_entries + kTile - 1) / kTile;
  const uint16_t* kb = p.k + b * p.k_sb + (int64_t)kvh * kD;
  const uint16_t* vb = p.v + b * p.v_sb + (int64_t)kvh * kD;

  // entry e (0..n_entries) -> (token, mask)
  auto entry = [&](int e, uint32_t& msk) -> int64_t {
    if (LIST) {
      int c = c_begin;
      int cnt = p.lcount[(int64_t)gg * p.n_chunks + c];
      while (e >= cnt && c + 1 < c_end) {
        e -= cnt;
        ++c;
        cnt = p.lcount[(int64_t)gg * p.n_chunks + c];
      }
      const uint2 x = p.list[(int64_t)gg * p.Lk_pad + c * kDecChunk + e];
      msk = x.y;
      return (int64_t)x.x;
    } else {
      const int64_t ve = e_begin + e;
      msk = allmask;
      return ve < p.n_sink_eff ? ve : p.win_lo + (ve - p.n_sink_eff);
    }
  };
  auto load_tile = [&](int it, int buf) {
    // 64 rows x 16 chunks for K and for V: 16 cp.async per thread
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int c = u * kDecThreads + tid;
      const int r = c >> 4, ch = c & 15;
      const int e = it * kTile + r;
      const bool ok = e < n_entries;
      uint32_t msk = 0;
      const int64_t j = ok ? entry(e, msk) : 0;
      cp_async16(dswz(sm.k[buf], r, ch), kb + j * p.k_sl + ch * 8, ok);
      cp_async16(dswz(sm.v[buf], r, ch), vb + j * p.v_sl + ch * 8, ok);
      if (ch == 0) sm.mask[buf][r] = ok ? msk : 0u;
    }
  };

  if (n_tiles > 0) load_tile(0, 0);
  cp_async_commit();
  __syncthreads();
  uint32_t qa[8][4];
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const int r = (lane & 7) + 8 * ((lane >> 3) & 1);
    ldmatrix_x4(qa[kk], dswz(sm.q, r, 2 * kk + (lane >> 4)));
  }
  float oacc[16][4];
#pragma unroll
  for (int d = 0; d < 16; ++d)
#pragma unroll
    for (int e = 0; e < 4; ++e) oacc[d][e] = 0.f;
  float mrow[2] = {-INFINITY, -INFINITY};
  float lrow[2] = {0.f, 0.f};

  for (int it = 0; it < n_tiles; ++it) {
    const int buf = it & 1;
    if (it + 1 < n_tiles) {
      load_tile(it + 1, buf ^ 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    // this warp: keys warp*16 .. +15 of the tile
    const int kw = warp * 16;
    float s[2][4];
#pragma unroll
    for (int e = 0; e < 4; ++e) { s[0][e] = 0.f; s[1][e] = 0.f; }
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const int q = lane >> 3;
      const int key = kw + (lane & 7) + 8 * (q >> 1);
      uint32_t r[4];
      ldmatrix_x4(r, dswz(sm.k[buf], key, 2 * kk + (q & 1)));
      mma16816(s[0], qa[kk], r[0], r[1], s[0]);
      mma16816(s[1], qa[kk], r[2], r[3], s[1]);
    }
    float tmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int n = 0; n < 2; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const bool hi = e >= 2;
        const int head = g + (hi ? 8 : 0);
        const int key = kw + n * 8 + 2 * t + (e & 1);
        const bool ok = (sm.mask[buf][key] >> head) & 1u;
        const float x = ok ? s[n][e] * p.scale_log2 : -INFINITY;
        s[n][e] = x;
        tmax[hi] = fmaxf(tmax[hi], x);
      }
    float alpha[2];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      tmax[hh] = quad_max(tmax[hh]);
      const float mnew = fmaxf(mrow[hh], tmax[hh]);
      alpha[hh] = (mrow[hh] == -INFINITY) ? 0.f : exp2f(mrow[hh] - mnew);
      mrow[hh] = mnew;
    }
    uint32_t pp[2][2];
    float ls[2] = {0.f, 0.f};
#pragma unroll
    for (int n = 0; n < 2; ++n) {
      float pr[4];
#pragma unroll
      for (int e = 0; e < 4; ++e)
        pr[e] = (s[n][e] == -INFINITY) ? 0.f : exp2f(s[n][e] - mrow[e >= 2]);
      pp[n][0] = pack_bf16x2(pr[0], pr[1]);
      pp[n][1] = pack_bf16x2(pr[2], pr[3]);
      ls[0] += bf16_lo(pp[n][0]) + bf16_hi(pp[n][0]);
      ls[1] += bf16_lo(pp[n][1]) + bf16_hi(pp[n][1]);
    }
    lrow[0] = lrow[0] * alpha[0] + ls[0];
    lrow[1] = lrow[1] * alpha[1] + ls[1];
#pragma unroll
    for (int d = 0; d < 16; ++d) {
      oacc[d][0] *= alpha[0];
      oacc[d][1] *= alpha[0];
      oacc[d][2] *= alpha[1];
      oacc[d][3] *= alpha[1];
    }
    const uint32_t pa[4] = {pp[0][0], pp[0][1], pp[1][0], pp[1][1]};
#pragma unroll
    for (int dp = 0; dp < 8; ++dp) {
      const int q = lane >> 3;
      const int key = kw + (lane & 7) + 8 * (q & 1);
      uint32_t r[4];
      ldmatrix_x4_trans(r, dswz(sm.v[buf], key, 2 * dp + (q >> 1)));
      mma16816(oacc[2 * dp], pa, r[0], r[1], oacc[2 * dp]);
      mma16816(oacc[2 * dp + 1], pa, r[2], r[3], oacc[2 * dp + 1]);
    }
    __syncthreads();
  }

  // ---- merge the 4 warps (each saw a quarter of every tile)
  lrow[0] = quad_sum(lrow[0]);
  lrow[1] = quad_sum(lrow[1]);
  if (t == 0) {
    sm.wm[warp][g] = mrow[0];
    sm.wm[warp][g + 8] = mrow[1];
    sm.wl[warp][g] = lrow[0];
    sm.wl[warp][g + 8] = lrow[1];
  }
#pragma unroll
  for (int d = 0; d < 16; ++d) {
    const int col = d * 8 + 2 * t;
    sm.wo[warp][g][col] = oacc[d][0];
    sm.wo[warp][g][col + 1] = oacc[d][1];
    sm.wo[warp][g + 8][col] = oacc[d][2];
    sm.wo[warp][g + 8][col + 1] = oacc[d][3];
  }
  __syncthreads();
  float* part = p.part + ((int64_t)gg * p.n_splits + split) * 16 * (2 + kD);
  for (int x = tid; x < 16 * kD; x += kDecThreads) {
    const int r = x / kD, d = x % kD;
    float M = -INFINITY;
    for (int w = 0; w < 4; ++w) M = fmaxf(M, sm.wm[w][r]);
    float o = 0.f, l = 0.f;
    if (M != -INFINITY) {
      for (int w = 0; w < 4; ++w) {
        const float f = (sm.wm[w][r] == -INFINITY) ? 0.f : exp2f(sm.wm[w][r] - M);
        o += f * sm.wo[w][r][d];
        l += f * sm.wl[w][r];
      }
    }
    part[r * (2 + kD) + 2 + d] = o;
    if (d == 0) {
      part[r * (2 + kD)] = M;
      part[r * (2 + kD) + 1] = l;
    }
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) sm.is_last = (atomicAdd(&p.mcount[gg], 1u) == (uint32_t)p.n_splits - 1);
  __syncthreads();
  if (!sm.is_last) return;
  __threadfence();

  // ---- last CTA of the group: merge splits in a fixed order
  const float* pg = p.part + (int64_t)gg * p.n_splits * 16 * (2 + kD);
  for (int x = tid; x < G * kD; x += kDecThreads) {
    const int r = x / kD, d = x % kD;
    float M = -INFINITY;
    for (int sp = 0; sp < p.n_splits; ++sp) M = fmaxf(M, __ldcg(pg + ((int64_t)sp * 16 + r) * (2 + kD)));
    float o = 0.f, l = 0.f;
    for (int sp = 0; sp < p.n_splits; ++sp) {
      const float* pr = pg + ((int64_t)sp * 16 + r) * (2 + kD);
      const float ms = __ldcg(pr);
      if (ms == -INFINITY) continue;
      const float f = exp2f(ms - M);
      l += f * __ldcg(pr + 1);
      o += f * __ldcg(pr + 2 + d);
    }
    const int h = kvh * G + r;
    p.o[b * p.o_sb + (int64_t)h * kD + d] = f32_to_bf16_bits(l > 0.f ? o / l : 0.f);
    if (d == 0 && p.lse != nullptr)
      p.lse[b * p.lse_sb + h] = l > 0.f ? (M + log2f(l)) * kLn2 : -INFINITY;
  }
  if (tid == 0) p.mcount[gg] = 0;
}

template <bool LIST>
rtp_status launch_dec_attn(const DecAttnParams& prm, int B, cudaStream_t s) {
  const size_t smem = sizeof(DecSmem);
  if (cudaFuncSetAttribute(dec_attn_kernel<LIST>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return RTP_ERR_CUDA;
  dim3 grid(prm.n_splits, B * prm.groups);
  if (grid.y > 65535) return RTP_ERR_UNSUPPORTED;
  TraceScope tr(LIST ? "dec_attn_list" : "dec_attn_range", s);
  dec_attn_kernel<LIST><<<grid, kDecThreads, smem, s>>>(prm);
  return check_cuda(cudaGetLastError());
}

void fill_dec_common(DecAttnParams& prm, const rtp_shape* shape, const rtp_view& q,
                     const rtp_view& k, const rtp_view& v, const rtp_view& o, float* lse,
                     float scale) {
  memset(&prm, 0, sizeof(prm));
  prm.q = static_cast<const uint16_t*>(q.ptr); prm.q_sb = q.stride_b;
  prm.k = static_cast<const uint16_t*>(k.ptr); prm.k_sb = k.stride_b; prm.k_sl = k.stride_l;
  prm.v = static_cast<const uint16_t*>(v.ptr); prm.v_sb = v.stride_b; prm.v_sl = v.stride_l;
  prm.o = static_cast<uint16_t*>(o.ptr); prm.o_sb = o.stride_b;
  prm.lse = lse;
  prm.lse_sb = shape->H;  // lse [B][H][Lq=1]
  prm.scale_log2 = scale * kLog2e;
  prm.G = shape->H / shape->Hkv;
}

// Range-mode decode over keys {j <= P : j < n_sink or j > P - window}.
rtp_status decode_range(const rtp_shape* shape, const int16_t* kv_heads, int n_groups,
                        int window, int n_sink, const rtp_view& q, const rtp_view& k,
                        const rtp_view& v, float scale, const rtp_view& o, float* lse,
                        void* ws, size_t ws_bytes, cudaStream_t s) {
  if (n_groups == 0 || shape->B == 0) return RTP_OK;
  const int64_t P = shape->q_pos0;
  const int64_t n_sink_eff = std::min<int64_t>((int64_t)n_sink, P + 1);
  int64_t win_lo = P - window + 1;
  if (win_lo < n_sink_eff) win_lo = n_sink_eff;
  const int64_t n_keys = n_sink_eff + (P - win_lo + 1);
  AttnDecodeWs L = range_decode_ws_layout(n_keys, shape->B * n_groups);
  if (ws == nullptr || ws_bytes < L.total) return RTP_ERR_WORKSPACE_TOO_SMALL;
  DecAttnParams prm;
  fill_dec_common(prm, shape, q, k, v, o, lse, scale);
  prm.groups = n_groups;
  prm.n_splits = L.n_splits;
  prm.P = P;
  prm.n_sink_eff = (int)n_sink_eff;
  prm.win_lo = win_lo;
  prm.n_keys = n_keys;
  prm.keys_per_split = kRangeKeysPerSplit;
  prm.part = reinterpret_cast<float*>(static_cast<char*>(ws) + L.part);
  prm.mcount = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + L.mcount);
  for (int i = 0; i < n_groups; ++i) prm.kvh[i] = kv_heads[i];
  if (cudaMemsetAsync(prm.mcount, 0, (size_t)shape->B * n_groups * sizeof(uint32_t), s) !=
      cudaSuccess)
    return RTP_ERR_CUDA;
  return launch_dec_attn<false>(prm, shape->B, s);
}

}  // namespace
}  // namespace rtp

using namespace rtp;

// ====================================================================== C ABI

extern "C" size_t rtp_workspace_size(rtp_op op, const rtp_shape* shape, const uint8_t* kv_role,
                                     int32_t k16_per_kv_head) {
  if (check_shape(shape) != RTP_OK) return kStatusBytes;
  HeadMap hm;
  const bool have_roles =
      kv_role != nullptr && make_headmap(shape, kv_role, k16_per_kv_head, &hm) == RTP_OK;
  switch (op) {
    case RTP_OP_SPARSE_DECODE:
      if (!have_roles) return kStatusBytes;
      return decode_ws_layout(shape, hm).total;
    case RTP_OP_LOCAL:
    case RTP_OP_DENSE: {
      if (shape->Lq != 1) return kStatusBytes;
      const int groups = (op == RTP_OP_DENSE) ? shape->Hkv : (have_roles ? hm.n_lkv : shape->Hkv);
      return range_decode_ws_layout(shape->q_pos0 + 1, shape->B * groups).total;
    }
    default:
      return kStatusBytes;
  }
}

extern "C" rtp_status rtp_local_attn(const rtp_shape* shape, const uint8_t* kv_role,
                                     int32_t window, int32_t n_sink, rtp_view q, rtp_view k,
                                     rtp_view v, float softmax_scale, rtp_view o, float* lse,
                                     void* ws, size_t ws_bytes, rtp_stream_t stream) {
  rtp_status st = check_shape(shape);
  if (st != RTP_OK) return st;
  if ((st = check_causal(shape)) != RTP_OK) return st;
  HeadMap hm;
  if ((st = make_headmap(shape, kv_role, 0, &hm)) != RTP_OK) return st;
  if (window < 1 || n_sink < 0) return RTP_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f) || !isfinite(softmax_scale)) return RTP_ERR_INVALID_ARG;
  const bool work = shape->B > 0 && shape->Lq > 0 && hm.n_lkv > 0;
  if (!work) return RTP_OK;
  if ((st = check_view(q, shape->H, kD, true)) != RTP_OK) return st;
  if ((st = check_view(k, shape->Hkv, kD, true)) != RTP_OK) return st;
  if ((st = check_view(v, shape->Hkv, kD, true)) != RTP_OK) return st;
  if ((st = check_view(o, shape->H, kD, true)) != RTP_OK) return st;
  if (ws == nullptr || ws_bytes < kStatusBytes) return RTP_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (shape->Lq == 1) {
    if (hm.G > 16 || (256 % hm.G) != 0) return RTP_ERR_UNSUPPORTED;
    return decode_range(shape, hm.lkv, hm.n_lkv, window, n_sink, q, k, v, softmax_scale, o, lse,
                        ws, ws_bytes, s);
  }
  return prefill_local(shape, hm, window, n_sink, q, k, v, softmax_scale, o, lse, s);
}

extern "C" rtp_status rtp_dense_attn(const rtp_shape* shape, rtp_view q, rtp_view k, rtp_view v,
                                     float softmax_scale, rtp_view o, float* lse, void* ws,
                                     size_t ws_bytes, rtp_stream_t stream) {
  rtp_status st = check_shape(shape);
  if (st != RTP_OK) return st;
  if ((st = check_causal(shape)) != RTP_OK) return st;
  if (!(softmax_scale > 0.f) || !isfinite(softmax_scale)) return RTP_ERR_INVALID_ARG;
  if (shape->B == 0 || shape->Lq == 0) return RTP_OK;
  if ((st = check_view(q, shape->H, kD, true)) != RTP_OK) return st;
  if ((st = check_view(k, shape->Hkv, kD, true)) != RTP_OK) return st;
  if ((st = check_view(v, shape->Hkv, kD, true)) != RTP_OK) return st;
  if ((st = check_view(o, shape->H, kD, true)) != RTP_OK) return st;
  if (ws == nullptr || ws_bytes < kStatusBytes) return RTP_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (shape->Lq == 1) {
    const int G = shape->H / shape->Hkv;
    if (G > 16 || (256 % G) != 0) return RTP_ERR_UNSUPPORTED;
    int16_t kvh[kMaxHeads];
    for (int g = 0; g < shape->Hkv; ++g) kvh[g] = (int16_t)g;
    const int window = (int)std::min<int64_t>(shape->q_pos0 + 1, 0x7FFFFFFF);
    return decode_range(shape, kvh, shape->Hkv, window, 0, q, k, v, softmax_scale, o, lse, ws,
                        ws_bytes, s);
  }
  return prefill_dense(shape, q, k, v, softmax_scale, o, lse, s);
}

extern "C" rtp_status rtp_sparse_attn_prefill(const rtp_shape* shape, const uint8_t* kv_role,
                                              int32_t k16_per_kv_head, rtp_view q, rtp_view k,
                                              rtp_view v, rtp_view q16, rtp_view k16,
                                              const float* thr, const int32_t* jtie,
                                              float softmax_scale, rtp_view o, float* lse,
                                              void* ws, size_t ws_bytes, rtp_stream_t stream) {
  rtp_status st = check_shape(shape);
  if (st != RTP_OK) return st;
  if ((st = check_causal(shape)) != RTP_OK) return st;
  HeadMap hm;
  if ((st = make_headmap(shape, kv_role, k16_per_kv_head, &hm)) != RTP_OK) return st;
  if (!(softmax_scale > 0.f) || !isfinite(softmax_scale)) return RTP_ERR_INVALID_ARG;
  if (shape->Lk > kMaxKeys) return RTP_ERR_UNSUPPORTED;
  const bool work = shape->B > 0 && shape->Lq > 0 && hm.n_ret > 0;
  if (!work) return RTP_OK;
  if (thr == nullptr || jtie == nullptr) return RTP_ERR_INVALID_ARG;
  if ((st = check_view(q, shape->H, kD, true)) != RTP_OK) return st;
  if ((st = check_view(k, shape->Hkv, kD, true)) != RTP_OK) return st;
  if ((st = check_view(v, shape->Hkv, kD, true)) != RTP_OK) return st;
  if ((st = check_view(o, shape->H, kD, true)) != RTP_OK) return st;
  if ((st = check_view(q16, hm.n_ret, kR, true)) != RTP_OK) return st;
  if ((st = check_view(k16, hm.H_k16, kR, true)) != RTP_OK) return st;
  if (ws == nullptr || ws_bytes < kStatusBytes) return RTP_ERR_WORKSPACE_TOO_SMALL;
  return prefill_sparse(shape, hm, q, k, v, q16, k16, thr, jtie, softmax_scale, o, lse,
                        reinterpret_cast<cudaStream_t>(stream));
}

extern "C" rtp_status rtp_sparse_attn_decode(const rtp_shape* shape, const uint8_t* kv_role,
                                             int32_t k16_per_kv_head, rtp_view q,
                                             rtp_view k_cache, rtp_view v_cache, rtp_view q16,
                                             rtp_view k16_cache, float p, float softmax_scale,
                                             rtp_view o, float* lse, float* thr, int32_t* jtie,
                                             int32_t* count, float* mass, void* ws,
                                             size_t ws_bytes, rtp_stream_t stream) {
  rtp_status st = check_shape(shape);
  if (st != RTP_OK) return st;
  if (shape->Lq != 1) return RTP_ERR_INVALID_ARG;
  if ((st = check_causal(shape)) != RTP_OK) return st;
  HeadMap hm;
  if ((st = make_headmap(shape, kv_role, k16_per_kv_head, &hm)) != RTP_OK) return st;
  if (!(p >= 0.f && p <= 1.f)) return RTP_ERR_INVALID_ARG;
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
  // the query position decides how many cache rows are keys
  rtp_shape sh = *shape;
  const int N = (int)(shape->q_pos0 + 1);
  const DecodeWs L = decode_ws_layout(&sh, hm);
  if (ws == nullptr || ws_bytes < L.total) return RTP_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  RowRes* rowres = reinterpret_cast<RowRes*>(w + L.rowres);
  float* scores = reinterpret_cast<float*>(w + L.scores);
  const int n_chunks = (N + kDecChunk - 1) / kDecChunk;

  // 1. scores (always: the compaction reads them even when p >= 1)
  {
    ScoreParams sp;
    sp.q16 = static_cast<const uint16_t*>(q16.ptr);
    sp.q16_sb = q16.stride_b;
    sp.k16 = static_cast<const uint16_t*>(k16_cache.ptr);
    sp.k16_sb = k16_cache.stride_b;
    sp.k16_sl = k16_cache.stride_l;
    sp.scores = scores;
    sp.cmax = reinterpret_cast<float*>(w + L.cmax);
    sp.N = N;
    sp.Lk_pad = L.Lk_pad;
    sp.n_chunks = L.n_chunks;
    sp.n_ret = hm.n_ret;
    sp.n_rkv = hm.n_rkv;
    sp.G = hm.G;
    sp.per_kv = k16_per_kv_head;
    sp.hist_m = reinterpret_cast<unsigned long long*>(w + L.hist_m);
    sp.hist_c = reinterpret_cast<uint32_t*>(w + L.hist_c);
    sp.zsum = reinterpret_cast<unsigned long long*>(w + L.zsum);
    sp.counter = reinterpret_cast<uint32_t*>(w + L.counter);
    sp.mcount = reinterpret_cast<uint32_t*>(w + L.mcount);
    const size_t smem = (size_t)hm.G * (kDecChunk + 4) * sizeof(float);
    if (cudaFuncSetAttribute(dec_score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return RTP_ERR_CUDA;
    dim3 grid(n_chunks, shape->B * hm.n_rkv);
    TraceScope tr("dec_score", s);
    dec_score_kernel<<<grid, kScoreThreads, smem, s>>>(sp);
    if ((st = check_cuda(cudaGetLastError())) != RTP_OK) return st;
  }
  // 2. threshold per row
  if (p >= 1.f) {
    TraceScope tr("dec_all", s);
    dec_all_kernel<<<(L.rows + 127) / 128, 128, 0, s>>>(rowres, L.rows, N, thr, jtie, count, mass);
  } else {
    HistParams hp;
    hp.scores = scores;
    hp.cmax = reinterpret_cast<const float*>(w + L.cmax);
    hp.hist_m = reinterpret_cast<unsigned long long*>(w + L.hist_m);
    hp.hist_c = reinterpret_cast<uint32_t*>(w + L.hist_c);
    hp.zsum = reinterpret_cast<unsigned long long*>(w + L.zsum);
    hp.counter = reinterpret_cast<uint32_t*>(w + L.counter);
    hp.rowres = rowres;
    hp.thr = thr;
    hp.jtie = jtie;
    hp.count = count;
    hp.mass = mass;
    hp.status = reinterpret_cast<DevStatus*>(w);
    hp.N = N;
    hp.Lk_pad = L.Lk_pad;
    hp.n_chunks = n_chunks;
    hp.cmax_stride = L.n_chunks;
    hp.p = p;
    dim3 grid((N + kDecHistChunk - 1) / kDecHistChunk, L.rows);
    TraceScope tr("dec_hist", s);
    dec_hist_kernel<<<grid, kHistThreads, 0, s>>>(hp);
  }
  if ((st = check_cuda(cudaGetLastError())) != RTP_OK) return st;
  // 3. compaction
  {
    CompactParams cp;
    cp.scores = scores;
    cp.rowres = rowres;
    cp.list = reinterpret_cast<uint2*>(w + L.list);
    cp.lcount = reinterpret_cast<int32_t*>(w + L.lcount);
    cp.N = N;
    cp.Lk_pad = L.Lk_pad;
    cp.n_chunks = n_chunks;
    cp.n_ret = hm.n_ret;
    cp.n_rkv = hm.n_rkv;
    cp.G = hm.G;
    dim3 grid(n_chunks, shape->B * hm.n_rkv);
    TraceScope tr("dec_compact", s);
    dec_compact_kernel<<<grid, kCompactThreads, 0, s>>>(cp);
    if ((st = check_cuda(cudaGetLastError())) != RTP_OK) return st;
  }
  // 4. attention over the kept union
  DecAttnParams prm;
  fill_dec_common(prm, shape, q, k_cache, v_cache, o, lse, softmax_scale);
  prm.groups = hm.n_rkv;
  prm.list = reinterpret_cast<const uint2*>(w + L.list);
  prm.lcount = reinterpret_cast<const int32_t*>(w + L.lcount);
  prm.Lk_pad = L.Lk_pad;
  prm.n_chunks = n_chunks;
  prm.chunks_per_split = kDecChunksPerSplit;
  prm.n_splits = (n_chunks + kDecChunksPerSplit - 1) / kDecChunksPerSplit;
  prm.part = reinterpret_cast<float*>(w + L.part);
  prm.mcount = reinterpret_cast<uint32_t*>(w + L.mcount);
  for (int i = 0; i < hm.n_rkv; ++i) prm.kvh[i] = hm.rkv[i];
  return launch_dec_attn<true>(prm, shape->B, s);
}

// ====================================================================== no-allocation variant
// Scratch for rtp_local_attn_decode_noalloc: split-KV partials and merge
// counters in a file-scope device array instead of a caller workspace.
namespace rtp {
namespace {

__device__ __align__(256) unsigned char g_noalloc_scratch[RTP_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the array on the current device (looked up once per device;
// in host code the symbol itself is only a host-side stand-in).
rtp_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return RTP_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return RTP_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return RTP_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return RTP_OK;
}

}  // namespace
}  // namespace rtp

extern "C" rtp_status rtp_local_attn_decode_noalloc(const rtp_shape* shape,
                                                    const uint8_t* kv_role, int32_t window,
                                                    int32_t n_sink, rtp_view q, rtp_view k,
                                                    rtp_view v, float softmax_scale, rtp_view o,
                                                    float* lse, rtp_stream_t stream) {
  rtp_status st = check_shape(shape);
  if (st != RTP_OK) return st;
  if (shape->Lq != 1) return RTP_ERR_INVALID_ARG;
  if ((st = check_causal(shape)) != RTP_OK) return st;
  HeadMap hm;
  if ((st = make_headmap(shape, kv_role, 0, &hm)) != RTP_OK) return st;
  if (window < 1 || n_sink < 0) return RTP_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f) || !isfinite(softmax_scale)) return RTP_ERR_INVALID_ARG;
  if (shape->B == 0 || hm.n_lkv == 0) return RTP_OK;
  if (hm.G > 16 || (256 % hm.G) != 0) return RTP_ERR_UNSUPPORTED;
  if ((st = check_view(q, shape->H, kD, true)) != RTP_OK) return st;
  if ((st = check_view(k, shape->Hkv, kD, true)) != RTP_OK) return st;
  if ((st = check_view(v, shape->Hkv, kD, true)) != RTP_OK) return st;
  if ((st = check_view(o, shape->H, kD, true)) != RTP_OK) return st;
  // the same key set decode_range visits
  const int64_t P = shape->q_pos0;
  const int64_t n_sink_eff = std::min<int64_t>((int64_t)n_sink, P + 1);
  int64_t win_lo = P - window + 1;
  if (win_lo < n_sink_eff) win_lo = n_sink_eff;
  const int64_t n_keys = n_sink_eff + (P - win_lo + 1);
  const size_t need = range_decode_ws_layout(n_keys, shape->B * hm.n_lkv).total;
  if (need > (size_t)RTP_NOALLOC_SCRATCH_BYTES) return RTP_ERR_SCRATCH_LIMIT;
  void* scratch = nullptr;
  if ((st = noalloc_scratch(&scratch)) != RTP_OK) return st;
  return decode_range(shape, hm.lkv, hm.n_lkv, window, n_sink, q, k, v, softmax_scale, o, lse,
                      scratch, (size_t)RTP_NOALLOC_SCRATCH_BYTES,
                      reinterpret_cast<cudaStream_t>(stream));
}
