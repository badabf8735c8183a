// select_prefill.cu -- exact dynamic top-p for causal prefill rows (rtp_topp_select).
//
// Rule ("Dynamic Top-p Selection Mechanism", Eq. 5, paper-graph-ui summary of
// arXiv 2605.16928): softmax the indexer scores of a query row, keep the
// shortest prefix of the keys in (score desc, index asc) order whose mass
// reaches p * Z.  The L x L score matrix is never stored: each CTA owns 64 query
// rows of one retrieval head and streams that head's k16 tiles (L2-resident)
// through several sweeps, recomputing Q16.K16^T on the tensor cores each time:
//
//   sweep 1  row max m                                   (1 compare / pair)
//   sweep 2  Z = sum exp(s - m) and a 64-bin mass histogram of the scores in
//            [c0, m], c0 = m - ln(N / (1 - p)) - 1 (keys below c0 can never be
//            kept: their total mass is < (1-p) Z)          (1 exp / pair)
//   sweep 3+ radix refinement inside the crossing bin on the composite key
//            (score key : 32 bits, 2^21-1-index : 21 bits), 6 bits per sweep,
//            until the crossing bin holds <= 64 keys; those are collected,
//            sorted and walked to the exact cut (a compare / pair).
//
// Masses are summed as 40-bit fixed point in 64-bit integers, so every sum is
// exact and independent of the order atomics land in: the selection is
// deterministic run to run.
#include "rtp_host.h"

namespace rtp {
namespace {

constexpr int kBM = 64;
constexpr int kBN = 64;
constexpr int kNB = 64;
constexpr int kCap = 64;
constexpr int kThreads = 128;
constexpr int kIdxBits = 21;
constexpr unsigned long long kIdxMask = (1ull << kIdxBits) - 1;
constexpr int kKeyBits = 32 + kIdxBits;  // 53

enum { ST_IDLE = 0, ST_REFINE = 1, ST_COLLECT = 2, ST_DONE = 3 };

struct SelParams {
  const uint16_t* q16;
  int64_t q16_sb, q16_sl;
  const uint16_t* k16;
  int64_t k16_sb, k16_sl;
  int Lq, Lk;
  int64_t q_pos0;
  int n_ret;
  float p;
  float* thr;
  int32_t* jtie;
  int32_t* count;
  float* mass;
  DevStatus* status;
  int16_t k16_slot[kMaxHeads];
};

struct SelSmem {
  uint16_t k16[2][kBN][kR];
  unsigned long long hm[kBM][kNB];
  uint32_t hc[kBM][kNB];
  unsigned long long cand[kBM][kCap];
  unsigned long long zf[kBM];
  unsigned long long acc_above[kBM];
  unsigned long long prefix[kBM];
  double T[kBM];
  float m[kBM], c0[kBM], scale[kBM];
  uint32_t cnt_above[kBM];
  int state[kBM], k0[kBM], pbits[kBM], ncand[kBM];
};

__device__ __forceinline__ float canon(float s) { return s + 0.0f; }  // -0 -> +0

__device__ __forceinline__ float mass_w(float s, float m) {
  return exp2f(__fmul_rn(__fsub_rn(s, m), kLog2e));
}

__device__ __forceinline__ int bin0_of(float s, float m, float scale) {
  const int b = (int)__fmul_rn(__fsub_rn(m, s), scale);
  return b < kNB - 1 ? b : kNB - 1;
}

__device__ __forceinline__ unsigned long long comp_key(float s, int j) {
  return ((unsigned long long)score_key(s) << kIdxBits) | (kIdxMask - (unsigned long long)j);
}

__device__ __forceinline__ float key_score(uint32_t key) {
  const uint32_t b = (key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key;
  return __uint_as_float(b);
}

__device__ __forceinline__ unsigned long long shfl_xor_u64(unsigned long long v, int o) {
  const uint32_t lo = __shfl_xor_sync(0xffffffffu, (uint32_t)v, o);
  const uint32_t hi = __shfl_xor_sync(0xffffffffu, (uint32_t)(v >> 32), o);
  return ((unsigned long long)hi << 32) | lo;
}

struct SelCtx {
  int b, hr, slot, m0, nrows, n_tiles, warp, lane, g, t;
  int rA, rB;          // CTA-local rows owned by this thread (g, g+8 of the warp)
  int64_t PA, PB;      // their positions
  bool vA, vB;         // rows exist
  int64_t warp_maxP;   // largest position among this warp's rows (-1: none)
  uint32_t qa[4];      // q16 A fragment
};

// Stream the k16 tiles 0..n_tiles-1 and call body(kt, s) with this warp's
// 16 x 64 score tile (s[nt][e]: row g (e<2) or g+8, key kt*64 + nt*8 + 2t + (e&1)).
template <class Body>
__device__ __forceinline__ void sweep(SelSmem& sm, const SelParams& p, const SelCtx& c,
                                      bool warp_active, Body&& body) {
  const int tid = threadIdx.x;
  const uint16_t* kbase = p.k16 + c.b * p.k16_sb + c.slot * kR;
  auto load = [&](int kt, int buf) {
    const int key = tid >> 1, ch = tid & 1;
    const int j = kt * kBN + key;
    const bool ok = j < p.Lk;
    const uint16_t* src = kbase + (int64_t)(ok ? j : 0) * p.k16_sl + ch * 8;
    cp_async16(smem_u32(&sm.k16[buf][key][(ch ^ ((key >> 2) & 1)) * 8]), src, ok);
  };
  load(0, 0);
  cp_async_commit();
  for (int kt = 0; kt < c.n_tiles; ++kt) {
    if (kt + 1 < c.n_tiles) {
      load(kt + 1, (kt + 1) & 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (warp_active && (int64_t)kt * kBN <= c.warp_maxP) {
      const int buf = kt & 1;
      float s[8][4];
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        const int q = c.lane >> 3;
        const int key = np * 16 + (c.lane & 7) + 8 * (q >> 1);
        const int ch = q & 1;
        uint32_t r[4];
        ldmatrix_x4(r, smem_u32(&sm.k16[buf][key][(ch ^ ((key >> 2) & 1)) * 8]));
        mma16816_zero(s[2 * np], c.qa, r[0], r[1]);
        mma16816_zero(s[2 * np + 1], c.qa, r[2], r[3]);
      }
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) s[nt][e] = canon(s[nt][e]);
      body(kt, s);
    }
    __syncthreads();
  }
}

// Crossing search over a descending histogram: the first bin where the running
// mass reaches T.  Returns the bin; updates acc/cnt with the bins above it.
__device__ __forceinline__ int crossing(const unsigned long long* hm, const uint32_t* hc, int nb,
                                        double T, unsigned long long& acc, uint32_t& cnt,
                                        uint32_t& n_in) {
  int last = -1;
  for (int b = 0; b < nb; ++b) {
    if (hc[b] == 0) continue;
    last = b;
    if ((double)(acc + hm[b]) >= T) {
      n_in = hc[b];
      return b;
    }
    acc += hm[b];
    cnt += hc[b];
  }
  // rounding left T out of reach: keep everything, i.e. the lowest non-empty bin
  if (last >= 0) {
    acc -= hm[last];
    cnt -= hc[last];
    n_in = hc[last];
  }
  return last;
}

__global__ void __launch_bounds__(kThreads) topp_select_kernel(const SelParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SelSmem& sm = *reinterpret_cast<SelSmem*>(smem_raw);
  SelCtx c;
  c.b = blockIdx.z;
  c.hr = blockIdx.y;
  c.slot = p.k16_slot[c.hr];
  const int tile = gridDim.x - 1 - blockIdx.x;  // heavy (late) tiles first
  c.m0 = tile * kBM;
  c.nrows = min(kBM, p.Lq - c.m0);
  const int tid = threadIdx.x;
  c.warp = tid >> 5;
  c.lane = tid & 31;
  c.g = c.lane >> 2;
  c.t = c.lane & 3;
  c.rA = c.warp * 16 + c.g;
  c.rB = c.rA + 8;
  c.vA = c.rA < c.nrows;
  c.vB = c.rB < c.nrows;
  c.PA = p.q_pos0 + c.m0 + c.rA;
  c.PB = p.q_pos0 + c.m0 + c.rB;
  const int wlast = min(c.warp * 16 + 15, c.nrows - 1);
  c.warp_maxP = (wlast >= c.warp * 16) ? p.q_pos0 + c.m0 + wlast : -1;
  const int64_t Plast = p.q_pos0 + c.m0 + c.nrows - 1;
  c.n_tiles = (int)((Plast + kBN) / kBN);

  // q16 A fragment: rows g / g+8, dims 2t..2t+1 and 2t+8..2t+9
  {
    const uint16_t* qb = p.q16 + c.b * p.q16_sb + (int64_t)c.hr * kR;
    auto ld = [&](int r, int d) -> uint32_t {
      if (r >= c.nrows) return 0u;
      return *reinterpret_cast<const uint32_t*>(qb + (int64_t)(c.m0 + r) * p.q16_sl + d);
    };
    c.qa[0] = ld(c.rA, 2 * c.t);
    c.qa[1] = ld(c.rB, 2 * c.t);
    c.qa[2] = ld(c.rA, 2 * c.t + 8);
    c.qa[3] = ld(c.rB, 2 * c.t + 8);
  }

  // ---------------------------------------------------------- sweep 1: max
  {
    float mx[2] = {-INFINITY, -INFINITY};
    sweep(sm, p, c, true, [&](int kt, float (&s)[8][4]) {
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int64_t j = (int64_t)kt * kBN + nt * 8 + 2 * c.t + (e & 1);
          const bool hi = e >= 2;
          const bool ok = hi ? (c.vB && j <= c.PB) : (c.vA && j <= c.PA);
          if (ok) mx[hi] = fmaxf(mx[hi], s[nt][e]);
        }
    });
    mx[0] = quad_max(mx[0]);
    mx[1] = quad_max(mx[1]);
    if (c.t == 0) {
      sm.m[c.rA] = mx[0];
      sm.m[c.rB] = mx[1];
    }
  }
  __syncthreads();
  if (tid < kBM) {
    const int r = tid;
    if (r < c.nrows) {
      const double N = (double)(p.q_pos0 + c.m0 + r + 1);
      const float m = sm.m[r];
      const float R = (float)(log(N / (1.0 - (double)p.p)) + 1.0);
      sm.c0[r] = m - R;
      sm.scale[r] = (float)kNB / R;
      sm.state[r] = ST_REFINE;
    } else {
      sm.state[r] = ST_IDLE;
    }
    sm.acc_above[r] = 0;
    sm.cnt_above[r] = 0;
    sm.ncand[r] = 0;
    sm.pbits[r] = 0;
    sm.prefix[r] = 0;
    for (int b = 0; b < kNB; ++b) {
      sm.hm[r][b] = 0;
      sm.hc[r][b] = 0;
    }
  }
  __syncthreads();

  // ---------------------------------------------------------- sweep 2: Z + level-0 histogram
  {
    const float mA = sm.m[c.rA], mB = sm.m[c.rB];
    const float cA = sm.c0[c.rA], cB = sm.c0[c.rB];
    const float sA = sm.scale[c.rA], sB = sm.scale[c.rB];
    unsigned long long z[2] = {0ull, 0ull};
    sweep(sm, p, c, true, [&](int kt, float (&s)[8][4]) {
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int64_t j = (int64_t)kt * kBN + nt * 8 + 2 * c.t + (e & 1);
          const bool hi = e >= 2;
          const bool ok = hi ? (c.vB && j <= c.PB) : (c.vA && j <= c.PA);
          if (!ok) continue;
          const float sv = s[nt][e];
          const float m = hi ? mB : mA;
          const unsigned long long f = mass_fixed40(mass_w(sv, m));
          z[hi] += f;
          if (sv >= (hi ? cB : cA)) {
            const int r = hi ? c.rB : c.rA;
            const int bin = bin0_of(sv, m, hi ? sB : sA);
            atomicAdd(&sm.hm[r][bin], f);
            atomicAdd(&sm.hc[r][bin], 1u);
          }
        }
    });
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      z[h] += shfl_xor_u64(z[h], 1);
      z[h] += shfl_xor_u64(z[h], 2);
    }
    if (c.t == 0) {
      sm.zf[c.rA] = z[0];
      sm.zf[c.rB] = z[1];
    }
  }
  __syncthreads();
  if (tid < c.nrows) {
    const int r = tid;
    const double T = (double)p.p * (double)sm.zf[r];
    sm.T[r] = T;
    unsigned long long acc = 0;
    uint32_t cnt = 0, n_in = 0;
    const int b = crossing(sm.hm[r], sm.hc[r], kNB, T, acc, cnt, n_in);
    sm.acc_above[r] = acc;
    sm.cnt_above[r] = cnt;
    sm.k0[r] = b;
    // composite-key prefix shared by every score this bin can hold
    const float m = sm.m[r], scale = sm.scale[r];
    const float hi_s = m - (float)b / scale, lo_s = m - (float)(b + 1) / scale;
    const float margin = 1e-5f * (fabsf(m) + (float)kNB / scale + 1.f);
    const unsigned long long kl = (unsigned long long)score_key(lo_s - margin) << kIdxBits;
    const unsigned long long kh =
        ((unsigned long long)score_key(hi_s + margin) << kIdxBits) | kIdxMask;
    const int pb = (kl == kh) ? kKeyBits : (__clzll(kl ^ kh) - (64 - kKeyBits));
    sm.pbits[r] = pb;
    sm.prefix[r] = pb > 0 ? (kh >> (kKeyBits - pb)) : 0ull;
    sm.state[r] = (n_in <= (uint32_t)kCap) ? ST_COLLECT : ST_REFINE;
    for (int bb = 0; bb < kNB; ++bb) {
      sm.hm[r][bb] = 0;
      sm.hc[r][bb] = 0;
    }
  }
  __syncthreads();

  // ---------------------------------------------------------- sweeps 3+: refine / collect
  for (int iter = 0; iter < 16; ++iter) {
    const int active = __syncthreads_or(tid < kBM && (sm.state[tid] == ST_REFINE ||
                                                      sm.state[tid] == ST_COLLECT));
    if (!active) break;
    int stA = sm.state[c.rA], stB = sm.state[c.rB];
    const bool wact = __any_sync(0xffffffffu, (stA == ST_REFINE || stA == ST_COLLECT) ||
                                                  (stB == ST_REFINE || stB == ST_COLLECT));
    const float mA = sm.m[c.rA], mB = sm.m[c.rB];
    const float cA = sm.c0[c.rA], cB = sm.c0[c.rB];
    const float sA = sm.scale[c.rA], sB = sm.scale[c.rB];
    const int kA = sm.k0[c.rA], kB = sm.k0[c.rB];
    const int pbA = sm.pbits[c.rA], pbB = sm.pbits[c.rB];
    const unsigned long long pxA = sm.prefix[c.rA], pxB = sm.prefix[c.rB];
    sweep(sm, p, c, wact, [&](int kt, float (&s)[8][4]) {
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const bool hi = e >= 2;
          const int st = hi ? stB : stA;
          if (st != ST_REFINE && st != ST_COLLECT) continue;
          const int64_t j = (int64_t)kt * kBN + nt * 8 + 2 * c.t + (e & 1);
          if (j > (hi ? c.PB : c.PA)) continue;
          const float sv = s[nt][e];
          if (sv < (hi ? cB : cA)) continue;
          const float m = hi ? mB : mA;
          if (bin0_of(sv, m, hi ? sB : sA) != (hi ? kB : kA)) continue;
          const unsigned long long ck = comp_key(sv, (int)j);
          const int pb = hi ? pbB : pbA;
          if (pb > 0 && (ck >> (kKeyBits - pb)) != (hi ? pxB : pxA)) continue;
          const int r = hi ? c.rB : c.rA;
          if (st == ST_COLLECT) {
            const int idx = atomicAdd(&sm.ncand[r], 1);
            if (idx < kCap) sm.cand[r][idx] = ck;
          } else {
            const int w = min(6, kKeyBits - pb);
            const int digit = (int)((ck >> (kKeyBits - pb - w)) & ((1ull << w) - 1));
            const int bin = (1 << w) - 1 - digit;
            atomicAdd(&sm.hm[r][bin], mass_fixed40(mass_w(sv, m)));
            atomicAdd(&sm.hc[r][bin], 1u);
          }
        }
    });
    __syncthreads();
    if (tid < kBM) {
      const int r = tid;
      const int st = sm.state[r];
      if (st == ST_COLLECT) {
        int n = sm.ncand[r];
        if (n > kCap) {
          set_status(p.status, RTP_ERR_DEVICE_TIMEOUT, 11);
          n = kCap;
        }
        unsigned long long* cd = sm.cand[r];
        for (int a = 1; a < n; ++a) {  // insertion sort, descending
          const unsigned long long x = cd[a];
          int q = a - 1;
          while (q >= 0 && cd[q] < x) {
            cd[q + 1] = cd[q];
            --q;
          }
          cd[q + 1] = x;
        }
        unsigned long long cum = sm.acc_above[r];
        const double T = sm.T[r];
        const float m = sm.m[r];
        int take = n;
        for (int a = 0; a < n; ++a) {
          cum += mass_fixed40(mass_w(key_score((uint32_t)(cd[a] >> kIdxBits)), m));
          if ((double)cum >= T) {
            take = a + 1;
            break;
          }
        }
        const unsigned long long last = cd[take - 1];
        const int i = c.m0 + r;
        const int64_t o = ((int64_t)c.b * p.n_ret + c.hr) * p.Lq + i;
        p.thr[o] = key_score((uint32_t)(last >> kIdxBits));
        p.jtie[o] = (int32_t)(kIdxMask - (last & kIdxMask));
        p.count[o] = (int32_t)(sm.cnt_above[r] + take);
        if (p.mass) p.mass[o] = (float)((double)cum / (double)sm.zf[r]);
        sm.state[r] = ST_DONE;
      } else if (st == ST_REFINE) {
        const int pb = sm.pbits[r];
        const int w = min(6, kKeyBits - pb);
        unsigned long long acc = sm.acc_above[r];
        uint32_t cnt = sm.cnt_above[r], n_in = 0;
        const int b = crossing(sm.hm[r], sm.hc[r], 1 << w, sm.T[r], acc, cnt, n_in);
        sm.acc_above[r] = acc;
        sm.cnt_above[r] = cnt;
        const int digit = (1 << w) - 1 - b;
        sm.prefix[r] = (sm.prefix[r] << w) | (unsigned long long)digit;
        sm.pbits[r] = pb + w;
        sm.state[r] = (n_in <= (uint32_t)kCap || pb + w >= kKeyBits) ? ST_COLLECT : ST_REFINE;
        for (int bb = 0; bb < kNB; ++bb) {
          sm.hm[r][bb] = 0;
          sm.hc[r][bb] = 0;
        }
      }
      sm.ncand[r] = 0;
    }
  }
}

// p >= 1: every causal key is kept; no scores are needed.
__global__ void topp_all_kernel(int n_ret, int Lq, int64_t q_pos0, int B, float* thr,
                                int32_t* jtie, int32_t* count, float* mass) {
  const int64_t n = (int64_t)B * n_ret * Lq;
  for (int64_t o = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; o < n;
       o += (int64_t)gridDim.x * blockDim.x) {
    const int i = (int)(o % Lq);
    thr[o] = -INFINITY;
    jtie[o] = (int32_t)(q_pos0 + i);
    count[o] = (int32_t)(q_pos0 + i + 1);
    if (mass) mass[o] = 1.f;
  }
}

}  // namespace
}  // namespace rtp

using namespace rtp;

extern "C" rtp_status rtp_topp_select(const rtp_shape* shape, const uint8_t* kv_role,
                                      int32_t k16_per_kv_head, rtp_view q16, rtp_view k16,
                                      float p, float* thr, int32_t* jtie, int32_t* count,
                                      float* mass, void* ws, size_t ws_bytes,
                                      rtp_stream_t stream) {
  rtp_status st = check_shape(shape);
  if (st != RTP_OK) return st;
  if ((st = check_causal(shape)) != RTP_OK) return st;
  HeadMap hm;
  if ((st = make_headmap(shape, kv_role, k16_per_kv_head, &hm)) != RTP_OK) return st;
  if (!(p >= 0.f && p <= 1.f)) return RTP_ERR_INVALID_ARG;
  if (shape->Lk > kMaxKeys) return RTP_ERR_UNSUPPORTED;
  const bool work = shape->B > 0 && shape->Lq > 0 && hm.n_ret > 0;
  if (!work) return RTP_OK;
  if (thr == nullptr || jtie == nullptr || count == nullptr) return RTP_ERR_INVALID_ARG;
  if (ws == nullptr || ws_bytes < kStatusBytes) return RTP_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (p >= 1.f) {
    TraceScope tr("topp_all", s);
    topp_all_kernel<<<592, 256, 0, s>>>(hm.n_ret, shape->Lq, shape->q_pos0, shape->B, thr,
                                        jtie, count, mass);
    return check_cuda(cudaGetLastError());
  }
  if ((st = check_view(q16, hm.n_ret, kR, true)) != RTP_OK) return st;
  if ((st = check_view(k16, hm.H_k16, kR, true)) != RTP_OK) return st;
  SelParams prm;
  prm.q16 = static_cast<const uint16_t*>(q16.ptr);
  prm.q16_sb = q16.stride_b;
  prm.q16_sl = q16.stride_l;
  prm.k16 = static_cast<const uint16_t*>(k16.ptr);
  prm.k16_sb = k16.stride_b;
  prm.k16_sl = k16.stride_l;
  prm.Lq = shape->Lq;
  prm.Lk = shape->Lk;
  prm.q_pos0 = shape->q_pos0;
  prm.n_ret = hm.n_ret;
  prm.p = p;
  prm.thr = thr;
  prm.jtie = jtie;
  prm.count = count;
  prm.mass = mass;
  prm.status = static_cast<DevStatus*>(ws);
  for (int i = 0; i < hm.n_ret; ++i) prm.k16_slot[i] = hm.ret_k16[i];
  const size_t smem = sizeof(SelSmem);
  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(topp_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return RTP_ERR_CUDA;
    attr_set = true;
  }
  dim3 grid((shape->Lq + kBM - 1) / kBM, hm.n_ret, shape->B);
  if (grid.y > 65535 || grid.z > 65535) return RTP_ERR_UNSUPPORTED;
  TraceScope tr("topp_select", s);
  topp_select_kernel<<<grid, kThreads, smem, s>>>(prm);
  return check_cuda(cudaGetLastError());
}
