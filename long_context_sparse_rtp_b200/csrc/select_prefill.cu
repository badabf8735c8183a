// select_prefill.cu -- exact dynamic top-p for causal prefill rows (rtp_topp_select).
//
// Rule ("Dynamic Top-p Selection Mechanism", Eq. 5, paper-graph-ui summary of
// arXiv 2605.16928): softmax the indexer scores of a query row, keep the
// shortest prefix of the keys in (score desc, index asc) order whose mass
// reaches p * Z.  The L x L score matrix is never stored.  A CTA owns 128 query
// rows of one retrieval head and sweeps that head's k16 rows (L2-resident)
// several times; every sweep recomputes the 128 x 128 score tiles
// S = Q16 . K16^T on the tensor cores (one tcgen05.mma, M = N = 128, K = 16,
// per tile, fp32 in TMEM).  Two epilogue threads per query row (TMEM lane r,
// key columns 0-63 and 64-127 of each tile) read the scores with tcgen05.ld;
// both derive the row's decisions identically from shared memory:
//
//   sweep 1  row max m and a lower bound Z_lo on Z = sum exp(s - m) (per 16 keys
//            the larger of exp(max - m) and the mass of every fourth key), 64
//            scores of a tile per TMEM wait
//   sweep 2  Z in a fixed order and a 32-bin mass histogram of the scores in
//            [m - R, m], R = min(ln(N / ((1 - p) Z_lo)), ln(N / (1 - p))) + 1/16:
//            keys below m - R + 1/16 are never kept (together they weigh less
//            than (1 - p) Z); the crossing bin k0 is where the mass from the top
//            reaches p Z
//   sweep 3+ per row, until its crossing range holds <= 32 keys, which are
//            collected, sorted and walked to the exact cut:
//            - level 1: 32 uniform score sub-bins of bin k0 (one sweep);
//            - then 5-bit digits of the composite key (score key : 32 bits,
//              2^21-1-index : 21 bits), one sweep each;
//            - a range of <= 8128 keys is instead parked once in the row's
//              global list, and its remaining digits are resolved over the
//              list, a warp per row, with no further sweep.
//            A sweep tests each key against the rows' ranges with one compare
//            (|s - mid| <= half) and queues the hits per warp (a chunk in which
//            no lane has two hits places them by one ballot, others by a prefix
//            sum); the queue is drained 32 hits at a time.  The list levels
//            load kListBatch entries per lane before compacting them in place.
//            Range counts are bounds taken from the bin sums (every key adds at
//            least a known amount); the count of keys above the final range is
//            exact.
//
// Histogram masses are kept relative to the top edge e of their bin: a key adds
// trunc(2^21 exp(s - e)) (a value in (exp(-w), 1] x 2^21, w the bin width) to
// its bin, so 32-bit shared-memory atomics per tile group, flushed into 64-bit
// sums, are exact and order-free; a bin's mass is its integer sum times
// exp(e - m) 2^-21, taken in fp64 in a fixed order.  Z is a fixed-order fp32
// tree per 16 keys summed in fp64.  The selection is deterministic run to run.
//
// Warp roles: warps 0-7 epilogue (warps w and w + 4 share TMEM lanes 32 (w & 3)
// .. +31, one column half each), warp 8 the TMA producer (Q16 tile once, K16
// tiles into a ring), warp 9 the MMA issuer (owns the 256 TMEM columns: two
// 128-column accumulators).
#include <cuda.h>

#include "rtp_host.h"
#include "tcgen05.cuh"
#include "tma.cuh"

namespace rtp {
namespace {

constexpr int kBM = 128;         // query rows per CTA (MMA M, TMEM lanes)
constexpr int kBN = 128;         // keys per tile (MMA N)
constexpr int kStages = 4;       // K16 tile ring
constexpr int kTileBytes = kBN * kR * 2;
constexpr int kNB = 32;          // histogram bins (5-bit digits)
constexpr int kDigit = 5;
constexpr int kCap = 32;         // candidates collected per row
constexpr int kGroup = 16;       // tiles per 32-bit bin-sum group: 16 x 64 keys x (2^21 + 1) < 2^32
constexpr int kMaxIter = 16;     // refine / collect sweeps (53 key bits / 5 + 1 suffice)
constexpr int kQueue = 64;       // per-warp queue of refine hits (drained at 32)
constexpr int kChunk = 16;       // keys per TMEM load and per unrolled body
constexpr double kRangePad = 1.0 / 16;  // level-0 range beyond the never-kept point
constexpr int kEpi = 256;        // epilogue threads: two per query row (column halves)
constexpr int kProdWarp = kEpi / 32, kMmaWarp = kEpi / 32 + 1;
constexpr int kThreads = kEpi + 64;
constexpr int kIdxBits = 21;
constexpr unsigned long long kIdxMask = (1ull << kIdxBits) - 1;
constexpr int kKeyBits = 32 + kIdxBits;  // 53
constexpr uint32_t kIdesc = idesc_bf16_f32(kBM, kBN);

// row states: REFINE1 = 32 uniform score sub-bins of the level-0 crossing bin,
// REFINE = 5 composite-key bits, COLLECT / LIST = gather the crossing range's keys
enum { ST_IDLE = 0, ST_REFINE1 = 1, ST_REFINE = 2, ST_COLLECT = 3, ST_DONE = 4, ST_LIST = 5 };
// Crossing-range keys a row may park in its global list.  A level's even and odd
// entries go to separate 32-bit bin sums, and the warp that reads the list moves
// them into the 64-bit sums after every kListFlush entries: <= 2032 keys x
// (2^21 + 1) < 2^32 in each copy between flushes.
constexpr int kListFlush = 4064;
constexpr int kListCap = 2 * kListFlush;
constexpr int kListBatch = 4;    // list entries per lane loaded together

struct SelParams {
  unsigned long long* lists;  // [slots][kBM][kListCap] crossing-bin keys, or null
  uint32_t* slot_mask;        // [SMs]: bit b = slot 2 sm + b in use
  int n_sm;
  int Lq;
  int64_t q_pos0;
  int n_ret;
  float p;
  int batch_coord_q, batch_coord_k;
  float* thr;
  int32_t* jtie;
  int32_t* count;
  float* mass;
  DevStatus* status;
  int16_t k16_slot[kMaxHeads];
};

struct SelSmem {
  uint8_t ktile[kStages][kTileBytes];  // 1024-byte aligned (the struct is placed so)
  uint8_t qtile[kBM * kR * 2];
  union {
    unsigned long long hw[kNB][kBM];   // per-row bin sums (units of 2^-21 of a bin edge), row fastest
    unsigned long long cand[kCap][kBM];
  } u;
  uint32_t wacc[2][kNB + 1][kBM];      // bin sums of the current tile group, one copy per
                                       // column half (the row's two threads); bin kNB
                                       // collects the keys below c0 and is never read
  union {
    float tab[kNB + 1][kBM];           // 2^21 exp(b / scale): level-0 bin b's edge factor
    struct {                           // refine sweeps: per-warp queues of prefilter hits
      float s[kEpi / 32][kQueue];
      uint32_t jl[kEpi / 32][kQueue];  // key index | owner lane << 21
    } q;
    struct {                           // parked-list levels: the state the warps read
      unsigned long long prefix[kBM];
      int pbits[kBM];
      int n[kBM];                      // entries of the row's compacted list
      int need[kBM];
      float m[kBM];
      float tk[kBM];
    } ls;
  } t;
  float mpart[2][kBM];
  double zpart[2][kBM];
  int ncnt[kBM];
  int nabove[kBM];                     // keys above the crossing range (exact)
  uint64_t full[kStages], empty[kStages], tfull[2], tempty[2], qfull, ctl;
  uint32_t tmem_base;
  int go;
  int gave_up;
  int slot;  // this CTA's candidate-list slot, -1 if none
};

__device__ __forceinline__ float ex2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}
// exp(s - m) for s <= m.
__device__ __forceinline__ float rel_w(float s, float m) {
  return ex2_ftz(__fmul_rn(__fsub_rn(s, m), kLog2e));
}
// trunc(x) for x in [0, 2^23): adding 2^23 with rounding toward zero leaves the
// integer part in the low mantissa bits.  Every use passes 2^21 exp(s - e) with
// s at most its bin's edge e up to rounding, so a key adds at most 2^21 + 1.
__device__ __forceinline__ uint32_t fixed_u(float x) {
  return __float_as_uint(__fadd_rz(x, 8388608.0f)) - 0x4B000000u;
}
// Level-0 bin of a score s <= m: floor((m - s) * scale), or kNB for a score at
// or below c0 = m - kNB / scale (adding 1.5 * 2^23 with rounding toward -inf
// leaves the floor in the low mantissa bits; larger or infinite products give
// larger integers, clamped).  Keys below c0 + 1 are never kept, so the rounding
// of that edge decides nothing.
__device__ __forceinline__ int bin0_of(float s, float m, float scale) {
  const int b = __float_as_int(__fadd_rd(__fmul_rn(__fsub_rn(m, s), scale), 12582912.0f)) -
                0x4B400000;
  return min(b, kNB);
}

__device__ __forceinline__ unsigned long long comp_key(float s, int j) {
  return ((unsigned long long)score_key(s) << kIdxBits) | (kIdxMask - (unsigned long long)j);
}

__device__ __forceinline__ float key_score(uint32_t key) {
  const uint32_t b = (key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key;
  return __uint_as_float(b);
}

// Crossing search over one row's descending histogram (column r of hw): the
// first non-empty bin b where base + factor(b) * (inner + hw[b]) reaches T.
// Returns the bin and its sum; adds the bins above it to inner (same-factor
// histograms) or base (a factor per bin).  Every key adds a positive amount to
// its bin, so a zero sum is an empty bin.
template <class Factor>
__device__ __forceinline__ int crossing(const SelSmem& sm, int r, int nb, double T, bool per_bin,
                                        Factor&& factor, double& base,
                                        unsigned long long& inner, unsigned long long& w_sel) {
  int last = -1;
  for (int b = 0; b < nb; ++b) {
    const unsigned long long wb = sm.u.hw[b][r];
    if (wb == 0ull) continue;
    last = b;
    const double f = factor(b);
    if (per_bin ? (base + f * (double)wb >= T) : (base + f * (double)(inner + wb) >= T)) {
      w_sel = wb;
      return b;
    }
    if (per_bin)
      base += f * (double)wb;
    else
      inner += wb;
  }
  // rounding left T out of reach: keep everything, i.e. the lowest non-empty bin
  w_sel = 0ull;
  if (last >= 0) {
    w_sel = sm.u.hw[last][r];
    if (per_bin)
      base -= factor(last) * (double)w_sel;
    else
      inner -= w_sel;
  }
  return last;
}

__device__ __forceinline__ void clear_row(SelSmem& sm, int r) {
#pragma unroll 8
  for (int b = 0; b < kNB; ++b) {
    sm.u.hw[b][r] = 0ull;
    sm.wacc[0][b][r] = 0u;
    sm.wacc[1][b][r] = 0u;
  }
}

// Moves the tile group's 32-bit bin sums (both copies) into the 64-bit ones.
__device__ __forceinline__ void flush_row(SelSmem& sm, int r) {
#pragma unroll 8
  for (int b = 0; b < kNB; ++b) {
    sm.u.hw[b][r] += (unsigned long long)sm.wacc[0][b][r] + sm.wacc[1][b][r];
    sm.wacc[0][b][r] = 0u;
    sm.wacc[1][b][r] = 0u;
  }
}

__device__ __forceinline__ float max16(const float (&v)[kChunk]) {
  // three-input maxima: 16 -> 6 -> 2 -> 1 (the max is exact in any order)
  const float a = max3f(v[0], v[1], v[2]), b = max3f(v[3], v[4], v[5]),
              c = max3f(v[6], v[7], v[8]), d = max3f(v[9], v[10], v[11]),
              e = max3f(v[12], v[13], v[14]);
  return fmaxf(max3f(a, b, c), max3f(d, e, v[15]));
}

// Level-1 sub-bin of a key of level-0 bin k0: the 32 uniform score sub-bins of
// that bin.  (m - s) * 32 scale is exactly 32 times the product bin0_of floors,
// so the sub-bins partition the bin.
__device__ __forceinline__ int sub1_of(float s, float m, float scale32, int k0) {
  const float x = fminf(__fmul_rn(__fsub_rn(m, s), scale32), 2097152.0f);
  const int b = __float_as_int(__fadd_rd(x, 12582912.0f)) - 0x4B400000 - kNB * k0;
  return min(max(b, 0), kNB - 1);
}

// Where a key stands against a row's crossing range (level-0 bin k0, level-1
// sub-bin k1 if k1 >= 0, composite-key prefix of pbits bits): -1 below, 0
// inside, 1 above.  The order is the one every histogram level used.
__device__ __forceinline__ int classify(float s, unsigned long long ck, float m, float scale,
                                        int k0, int k1, int pbits, unsigned long long prefix) {
  const int b0 = bin0_of(s, m, scale);
  if (b0 != k0) return b0 < k0 ? 1 : -1;
  if (k1 >= 0) {
    const int b1 = sub1_of(s, m, scale * (float)kNB, k0);
    if (b1 != k1) return b1 < k1 ? 1 : -1;
  }
  if (pbits > 0) {
    const unsigned long long px = ck >> (kKeyBits - pbits);
    if (px != prefix) return px > prefix ? 1 : -1;
  }
  return 0;
}

enum { MODE_SUB1 = 0, MODE_DIGIT = 1, MODE_COLLECT = 2, MODE_PARK = 3 };

// v[i] for a run-time i in [0, 16): a four-level select tree on the bits of i
// (registers cannot be indexed at run time).
__device__ __forceinline__ float pick16(const float (&v)[kChunk], int i) {
  float a[8], b[4];
#pragma unroll
  for (int k = 0; k < 8; ++k) a[k] = (i & 1) ? v[2 * k + 1] : v[2 * k];
#pragma unroll
  for (int k = 0; k < 4; ++k) b[k] = (i & 2) ? a[2 * k + 1] : a[2 * k];
  const float c0 = (i & 4) ? b[1] : b[0], c1 = (i & 4) ? b[3] : b[2];
  return (i & 8) ? c1 : c0;
}

// Processes the first n (<= 32) queued prefilter hits of this warp, one per
// lane, for the owning row (whose state is fetched from the owner lane):
// MODE_SUB1 adds the key to its level-1 sub-bin, MODE_DIGIT to its digit bin
// (the next w composite-key bits), MODE_COLLECT makes it a candidate,
// MODE_PARK stores it in the row's global list; the last two count the keys
// above the range up to hic (the sweep counts those past it).  Histogram sums go to this warp's column-half copy.
// Called by all 32 lanes.
__device__ __noinline__ void drain_hits(SelSmem& sm, unsigned long long* list, int wq, int n,
                                        int row0, int g, float m, float scale, int k0, int k1,
                                        int pbits, unsigned long long prefix, int w, float tk,
                                        int mode, float hic) {
  const int lane = threadIdx.x & 31;
  const bool has = lane < n;
  const float s = has ? sm.t.q.s[wq][lane] : 0.f;
  const uint32_t jl = has ? sm.t.q.jl[wq][lane] : 0u;
  const int owner = (int)(jl >> 21), j = (int)(jl & 0x1FFFFFu);
  const float om = __shfl_sync(0xffffffffu, m, owner);
  const float osc = __shfl_sync(0xffffffffu, scale, owner);
  const int ok0 = __shfl_sync(0xffffffffu, k0, owner);
  const int ok1 = __shfl_sync(0xffffffffu, k1, owner);
  const int opb = __shfl_sync(0xffffffffu, pbits, owner);
  const uint32_t opl = __shfl_sync(0xffffffffu, (uint32_t)prefix, owner);
  const uint32_t oph = __shfl_sync(0xffffffffu, (uint32_t)(prefix >> 32), owner);
  const int ow = __shfl_sync(0xffffffffu, w, owner);
  const float otk = __shfl_sync(0xffffffffu, tk, owner);
  const int omode = __shfl_sync(0xffffffffu, mode, owner);
  const float ohic = __shfl_sync(0xffffffffu, hic, owner);
  if (!has) return;
  const int r = row0 + owner;
  if (omode == MODE_SUB1) {
    if (bin0_of(s, om, osc) != ok0) return;
    const int b1 = sub1_of(s, om, osc * (float)kNB, ok0);
    atomicAdd(&sm.wacc[g][b1][r], fixed_u(__fmul_rn(rel_w(s, om), otk)));
    return;
  }
  const unsigned long long ck = comp_key(s, j);
  const int c = classify(s, ck, om, osc, ok0, ok1, opb, ((unsigned long long)oph << 32) | opl);
  if (omode == MODE_DIGIT) {
    if (c != 0) return;
    const int digit = (int)((ck >> (kKeyBits - opb - ow)) & ((1ull << ow) - 1));
    atomicAdd(&sm.wacc[g][(1 << ow) - 1 - digit][r], fixed_u(__fmul_rn(rel_w(s, om), otk)));
  } else if (c > 0) {  // keys past hic were counted by the sweep
    if (s <= ohic) atomicAdd(&sm.nabove[r], 1);
  } else if (c == 0) {
    const int slot_c = atomicAdd(&sm.ncnt[r], 1);
    if (omode == MODE_PARK) {
      if (slot_c < kListCap) list[(size_t)r * kListCap + slot_c] = ck;
    } else if (slot_c < kCap) {
      sm.u.cand[slot_c][r] = ck;
    }
  }
}

// The composite-key prefix shared by every score in [lo_s, hi_s] (widened by
// the margin that covers the fp32 rounding of the bin edges).
__device__ __forceinline__ void range_prefix(float lo_s, float hi_s, float margin, int& pbits,
                                             unsigned long long& prefix) {
  const unsigned long long kl = (unsigned long long)score_key(lo_s - margin) << kIdxBits;
  const unsigned long long kh = ((unsigned long long)score_key(hi_s + margin) << kIdxBits) | kIdxMask;
  pbits = (kl == kh) ? kKeyBits : (__clzll(kl ^ kh) - (64 - kKeyBits));
  prefix = pbits > 0 ? (kh >> (kKeyBits - pbits)) : 0ull;
}

// Score interval that holds every key of a row's crossing range (level-0 bin
// k0, level-1 sub-bin k1 if k1 >= 0, composite prefix), widened by the margin.
__device__ __forceinline__ void refine_range(float m, float scale, float margin, int k0, int k1,
                                             int pbits, unsigned long long prefix, float& lo,
                                             float& hi) {
  if (k1 >= 0) {
    const float s32 = scale * (float)kNB;
    lo = m - (float)(kNB * k0 + k1 + 1) / s32 - margin;
    hi = m - (float)(kNB * k0 + k1) / s32 + margin;
  } else {
    lo = m - (float)(k0 + 1) / scale - margin;
    hi = m - (float)k0 / scale + margin;
  }
  if (pbits > 0) {
    uint32_t k_lo, k_hi;
    if (pbits >= 32) {
      k_lo = k_hi = (uint32_t)(prefix >> (pbits - 32));
    } else {
      k_lo = (uint32_t)(prefix << (32 - pbits));
      k_hi = k_lo | ((1u << (32 - pbits)) - 1u);
    }
    float a = key_score(k_lo), c = key_score(k_hi);
    if (a != a) a = -INFINITY;  // key ranges that reach NaN encodings
    if (c != c) c = INFINITY;
    lo = fmaxf(lo, a);
    hi = fminf(hi, c);
  }
}

__global__ void __launch_bounds__(kThreads, 2)
    topp_select_kernel(const __grid_constant__ CUtensorMap qmap,
                       const __grid_constant__ CUtensorMap kmap, const SelParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SelSmem& sm = *reinterpret_cast<SelSmem*>(smem_raw +
                                             ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = blockIdx.z, hr = blockIdx.y;
  const int slot = p.k16_slot[hr];
  const int tile = gridDim.x - 1 - blockIdx.x;  // heavy (late) row blocks first
  const int m0 = tile * kBM;
  const int nrows = min(kBM, p.Lq - m0);
  const int64_t Plast = p.q_pos0 + m0 + nrows - 1;
  const int n_tiles = (int)((Plast + kBN) / kBN);

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.tfull[i], 1);
      mbar_init(&sm.tempty[i], kEpi / 32);
    }
    mbar_init(&sm.qfull, 1);
    mbar_init(&sm.ctl, 1);
    sm.gave_up = 0;
    sm.go = 0;
    fence_mbar_init();
    // a candidate-list slot of this SM (at most two CTAs are resident per SM)
    sm.slot = -1;
    if (p.lists != nullptr) {
      uint32_t smid;
      asm volatile("mov.u32 %0, %%smid;\n" : "=r"(smid));
      if ((int)smid < p.n_sm)
        for (int b2 = 0; b2 < 2 && sm.slot < 0; ++b2)
          if ((atomicOr(&p.slot_mask[smid], 1u << b2) & (1u << b2)) == 0u)
            sm.slot = (int)smid * 2 + b2;
    }
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&sm.tmem_base, 2 * kBN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* gave_up = &sm.gave_up;
  volatile int* go = &sm.go;

  if (warp == kProdWarp) {  // ------------------------------------- TMA producer
    if (lane == 0) {
      bool ok = true;
      int stage = 0, n_issued = 0;
      uint32_t sph = 0;
      mbar_arrive_expect_tx(&sm.qfull, (uint32_t)(kBM * kR * 2));
      tma_load_4d(sm.qtile, &qmap, 0, hr, m0, b * p.batch_coord_q, &sm.qfull);
      for (int sweep = 0; ok; ++sweep) {
        if (sweep >= 2) {  // another sweep only if some row still needs one
          ok = mbar_wait(&sm.ctl, (uint32_t)(sweep - 2) & 1u, gave_up);
          if (!ok || *go == 0) break;
        }
        for (int kt = 0; kt < n_tiles; ++kt) {
          if (!mbar_wait(&sm.empty[stage], sph ^ 1u, gave_up)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&sm.full[stage], (uint32_t)kTileBytes);
          tma_load_4d(sm.ktile[stage], &kmap, 0, slot, kt * kBN, b * p.batch_coord_k,
                      &sm.full[stage]);
          ++n_issued;
          if (++stage == kStages) {
            stage = 0;
            sph ^= 1u;
          }
        }
      }
      if (!ok) set_status(p.status, RTP_ERR_DEVICE_TIMEOUT, 12);
      // every copy in flight lands before the CTA may exit
      for (int k = max(0, n_issued - kStages); k < n_issued; ++k)
        mbar_wait_drain(&sm.full[k % kStages], (uint32_t)(k / kStages) & 1u);
      mbar_wait_drain(&sm.qfull, 0u);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {  // ------------------------------- MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(&sm.qfull, 0u, gave_up);
      const uint64_t adesc = sdesc_k_sw32(smem_u32(sm.qtile), 256);
      int stage = 0;
      uint32_t sph = 0, tcount = 0;
      for (int sweep = 0; ok; ++sweep) {
        if (sweep >= 2) {
          ok = mbar_wait(&sm.ctl, (uint32_t)(sweep - 2) & 1u, gave_up);
          if (!ok || *go == 0) break;
        }
        for (int kt = 0; kt < n_tiles; ++kt) {
          const int buf = (int)(tcount & 1u);
          if (!mbar_wait(&sm.full[stage], sph, gave_up) ||
              !mbar_wait(&sm.tempty[buf], ((tcount >> 1) & 1u) ^ 1u, gave_up)) {
            ok = false;
            break;
          }
          tc_fence_after();
          mma_bf16_ss(tmem + (uint32_t)(buf * kBN), adesc,
                      sdesc_k_sw32(smem_u32(sm.ktile[stage]), 256), kIdesc, false);
          mma_commit(&sm.empty[stage]);  // the K16 stage is free once the MMA has read it
          mma_commit(&sm.tfull[buf]);    // the accumulator is ready
          ++tcount;
          if (++stage == kStages) {
            stage = 0;
            sph ^= 1u;
          }
        }
      }
      if (!ok) set_status(p.status, RTP_ERR_DEVICE_TIMEOUT, 13);
      if (tcount > 0)  // the last MMA is complete before TMEM is released
        mbar_wait_drain(&sm.tfull[(tcount - 1) & 1u], ((tcount - 1) >> 1) & 1u);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ epilogue: two threads per row
    // Thread (r, g) reads TMEM lane r, columns 64 g .. 64 g + 63 of every tile.
    // Per-row decisions are computed identically by both from shared memory;
    // g == 0 clears, flushes and writes the outputs.
    const int r = tid & (kBM - 1), g = tid >> 7;
    const bool valid = r < nrows;
    const int64_t P = valid ? p.q_pos0 + m0 + r : -1;
    const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)(g * 64);
    uint32_t tcount = 0;
    bool ok = true;
    auto ebar = [] { named_bar(1, kEpi); };
    // one pass over the key tiles: body(j0, v) sees keys j0 .. j0 + 15 of this row
    // (keys past its causal limit read as -inf); with hist, each tile group's
    // 32-bit bin sums move to the 64-bit ones (rows with row_hist)
    auto sweep = [&](auto&& body, bool hist, bool row_hist) {
      for (int kt = 0; kt < n_tiles; ++kt) {
        const int buf = (int)(tcount & 1u);
        ok = ok && mbar_wait_warp(&sm.tfull[buf], (tcount >> 1) & 1u, gave_up);
        tc_fence_after();
        if (ok) {
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            float v[kChunk];
            const int j0 = kt * kBN + g * 64 + c * kChunk;
            tmem_ld16(lane_addr + (uint32_t)(buf * kBN + c * kChunk), v);
            if ((int64_t)j0 + kChunk - 1 > P) {
#pragma unroll
              for (int i = 0; i < kChunk; ++i)
                if ((int64_t)(j0 + i) > P) v[i] = -INFINITY;
            }
            body(j0, v);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.tempty[buf]);
        ++tcount;
        if (hist && ((kt & (kGroup - 1)) == kGroup - 1 || kt == n_tiles - 1)) {
          ebar();
          if (g == 0 && row_hist) flush_row(sm, r);
          ebar();
        }
      }
    };

    // ---- sweep 1: the row max m, and a lower bound on Z = sum exp(s - m): each
    // thread keeps a running max mz, moved once per tile to the max of its 64
    // keys there, and zs, a sum over its 16-key chunks of the larger of two
    // partial masses, exp(chunk max - mz) and the mass of every fourth key (both
    // at most the chunk's mass).  The tile's 64 scores come with one TMEM wait
    // and its four chunks are independent.
    float mz = -INFINITY, zs = 0.f;
    for (int kt = 0; kt < n_tiles; ++kt) {
      const int buf = (int)(tcount & 1u);
      ok = ok && mbar_wait_warp(&sm.tfull[buf], (tcount >> 1) & 1u, gave_up);
      tc_fence_after();
      if (ok) {
        uint32_t rr[2][32];
        tmem_ld32_nowait(lane_addr + (uint32_t)(buf * kBN), rr[0]);
        tmem_ld32_nowait(lane_addr + (uint32_t)(buf * kBN + 32), rr[1]);
        tmem_wait_ld();
        float v[4][kChunk];
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int i = 0; i < kChunk; ++i) {
            reg_fence(rr[c >> 1][(c & 1) * kChunk + i]);
            v[c][i] = __uint_as_float(rr[c >> 1][(c & 1) * kChunk + i]);
          }
        const int64_t jt0 = (int64_t)kt * kBN + g * 64;
        if (jt0 + 63 > P) {  // keys past the causal limit read as -inf
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int i = 0; i < kChunk; ++i)
              if (jt0 + c * kChunk + i > P) v[c][i] = -INFINITY;
        }
        float cm[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) cm[c] = max16(v[c]);
        const float tmx = fmaxf(fmaxf(cm[0], cm[1]), fmaxf(cm[2], cm[3]));
        if (tmx > mz) {  // rescale to the new running max (rare after the first tiles)
          zs = mz > -INFINITY ? zs * rel_w(mz, tmx) : 0.f;
          mz = tmx;
        }
        if (mz > -INFINITY) {
          float t[4];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const float a = __fadd_rn(__fadd_rn(rel_w(v[c][0], mz), rel_w(v[c][4], mz)),
                                      __fadd_rn(rel_w(v[c][8], mz), rel_w(v[c][12], mz)));
            t[c] = fmaxf(a, rel_w(cm[c], mz));
          }
          zs = __fadd_rn(__fadd_rn(zs, __fadd_rn(t[0], t[1])), __fadd_rn(t[2], t[3]));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.tempty[buf]);
      ++tcount;
    }
    sm.mpart[g][r] = mz;
    sm.zpart[g][r] = (double)zs;
    ebar();
    const float m = fmaxf(sm.mpart[0][r], sm.mpart[1][r]);
    float scale = 1.f, margin = 0.f;
    if (valid) {
      // A key below m - ln(N / ((1 - p) Z)) is never kept: all such keys weigh
      // less than (1 - p) Z together, so the keys above that point already pass
      // p Z.  Z is taken from below (the partial masses, and a 1e-3 margin for
      // the fp32 sums and ex2.approx), which only widens the range; R adds
      // kRangePad, so the cut lies at least that far above the range's lower
      // edge, far beyond the rounding of the bin arithmetic there.
      double zl = 0.0;
      for (int h = 0; h < 2; ++h)
        if (sm.mpart[h][r] > -INFINITY) zl += sm.zpart[h][r] * exp((double)(sm.mpart[h][r] - m));
      zl = fmax(zl * (1.0 - 1e-3), 1e-30);
      const double N = (double)(P + 1);
      const double r_loose = log(N / (1.0 - (double)p.p)) + kRangePad;  // Z >= 1
      const float R = (float)fmin(log(N / ((1.0 - (double)p.p) * zl)) + kRangePad, r_loose);
      scale = (float)kNB / R;
      margin = 1e-5f * (fabsf(m) + R + 1.f);
    }
    if (g == 0) {
      clear_row(sm, r);
      for (int bb = 0; bb <= kNB; ++bb) sm.t.tab[bb][r] = 2097152.0f * expf((float)bb / scale);
    }
    ebar();

    // ---- sweep 2: Z and the level-0 histogram over [c0, m]; a key in bin b adds
    // trunc(2^21 exp(s - m) exp(b / scale)) = trunc(2^21 exp(s - edge_b))
    double Zp = 0.0;
    sweep(
        [&](int, float (&v)[kChunk]) {
          if (!valid) return;
          // two keys per packed instruction, each lane rounded as the scalar
          // forms: rel_w and bin0_of from one difference (exp2(-(m - s) log2 e)
          // is exp2((s - m) log2 e) bit for bit), fixed_u as add.rz of 2^23
          const unsigned long long m2 = f2_pack(m, m), nl2 = f2_pack(-kLog2e, -kLog2e),
                                   sc2 = f2_pack(scale, scale),
                                   fl2 = f2_pack(12582912.0f, 12582912.0f),
                                   tz2 = f2_pack(8388608.0f, 8388608.0f);
          unsigned long long ee[kChunk / 2];
          int bb[kChunk];
#pragma unroll
          for (int k = 0; k < kChunk / 2; ++k) {
            const unsigned long long dm = f2_sub(m2, f2_pack(v[2 * k], v[2 * k + 1]));
            float a0, a1, y0, y1;
            f2_unpack(f2_mul(dm, nl2), a0, a1);
            ee[k] = f2_pack(ex2_ftz(a0), ex2_ftz(a1));
            f2_unpack(f2_add_rm(f2_mul(dm, sc2), fl2), y0, y1);
            bb[2 * k] = min(__float_as_int(y0) - 0x4B400000, kNB);  // kNB: below c0, never read
            bb[2 * k + 1] = min(__float_as_int(y1) - 0x4B400000, kNB);
          }
          float t[kChunk];  // every edge factor is read before the first store
#pragma unroll
          for (int i = 0; i < kChunk; ++i) t[i] = sm.t.tab[bb[i]][r];
          // no-return atomics: the stores of one chunk need not wait for each other
#pragma unroll
          for (int k = 0; k < kChunk / 2; ++k) {
            float f0, f1;
            f2_unpack(f2_add_rz(f2_mul(ee[k], f2_pack(t[2 * k], t[2 * k + 1])), tz2), f0, f1);
            atomicAdd(&sm.wacc[g][bb[2 * k]][r], __float_as_uint(f0) - 0x4B000000u);
            atomicAdd(&sm.wacc[g][bb[2 * k + 1]][r], __float_as_uint(f1) - 0x4B000000u);
          }
          // the fixed-order tree e[i] += e[i + w], w = 8, 4, 2, 1, on the pairs
#pragma unroll
          for (int w = kChunk / 4; w >= 1; w >>= 1)
#pragma unroll
            for (int k = 0; k < w; ++k) ee[k] = f2_add(ee[k], ee[k + w]);
          float z0, z1;
          f2_unpack(ee[0], z0, z1);
          Zp += (double)__fadd_rn(z0, z1);
        },
        true, valid);
    sm.zpart[g][r] = Zp;
    ebar();
    const double Z = sm.zpart[0][r] + sm.zpart[1][r];
    double T = 0.0, base = 0.0, fk = 0.0;  // fk: mass of one unit of bin k0's sums
    unsigned long long inner = 0ull, prefix = 0ull;
    int k0 = 0, k1 = -1, pbits = 0, state = ST_IDLE;
    float tk = 0.f;    // 2^21 exp(k0 / scale)
    float umin = 1.f;  // least amount one key of the current range adds
    unsigned long long n_cur = 0ull;  // bound on the keys of the current range
    unsigned long long* const lists =
        sm.slot >= 0 ? p.lists + (size_t)sm.slot * kBM * kListCap : nullptr;
    // upper bound on the keys of a range from its sum: every key adds >= umin
    auto bound = [&](unsigned long long wsum) {
      return (unsigned long long)((double)wsum / (double)umin);
    };
    // a range of <= kCap keys is collected, of <= kListCap parked once in the
    // row's global list; a larger one is refined by another sweep
    auto next_state = [&](unsigned long long n, bool at_level0) {
      if (n <= (unsigned long long)kCap || pbits >= kKeyBits) return (int)ST_COLLECT;
      if (lists != nullptr && n <= (unsigned long long)kListCap) return (int)ST_LIST;
      return at_level0 ? (int)ST_REFINE1 : (int)ST_REFINE;
    };
    if (valid) {
      T = (double)p.p * Z;
      unsigned long long wsel = 0ull;
      auto f0 = [&](int bb) { return 1.0 / (double)sm.t.tab[bb][r]; };
      k0 = crossing(sm, r, kNB, T, true, f0, base, inner, wsel);
      if (k0 < 0) {  // cannot happen: the max key is in bin 0
        set_status(p.status, RTP_ERR_DEVICE_TIMEOUT, 16);
        k0 = 0;
      }
      tk = sm.t.tab[k0][r];
      fk = f0(k0);
      umin = fmaxf(2097152.0f * expf(-1.0f / scale) * (1.0f - 1.0f / 1024.0f) - 1.0f, 1.0f);
      n_cur = bound(wsel);
      range_prefix(m - (float)(k0 + 1) / scale, m - (float)k0 / scale, margin, pbits, prefix);
      state = next_state(n_cur, true);
    }
    ebar();
    if (g == 0) clear_row(sm, r);

    // sort the row's <= kCap candidates (smem) and walk them to the exact cut
    auto finish_row = [&]() {
      int n = sm.ncnt[r];
      if (n > kCap) {
        set_status(p.status, RTP_ERR_DEVICE_TIMEOUT, 11);
        n = kCap;
      }
      const int i = m0 + r;
      const int64_t o = ((int64_t)b * p.n_ret + hr) * p.Lq + i;
      if (n == 0) {  // cannot happen for a consistent histogram; keep every key
        set_status(p.status, RTP_ERR_DEVICE_TIMEOUT, 15);
        p.thr[o] = -INFINITY;
        p.jtie[o] = (int32_t)P;
        p.count[o] = (int32_t)(P + 1);
        if (p.mass) p.mass[o] = 1.f;
        return;
      }
      for (int a = 1; a < n; ++a) {  // insertion sort, descending
        const unsigned long long x = sm.u.cand[a][r];
        int q = a - 1;
        while (q >= 0 && sm.u.cand[q][r] < x) {
          sm.u.cand[q + 1][r] = sm.u.cand[q][r];
          --q;
        }
        sm.u.cand[q + 1][r] = x;
      }
      unsigned long long acc = inner;
      double cum = base;
      int take = n;
      for (int a = 0; a < n; ++a) {
        const float sa = key_score((uint32_t)(sm.u.cand[a][r] >> kIdxBits));
        acc += fixed_u(__fmul_rn(rel_w(sa, m), tk));
        cum = base + fk * (double)acc;
        if (cum >= T) {
          take = a + 1;
          break;
        }
      }
      const unsigned long long last = sm.u.cand[take - 1][r];
      p.thr[o] = key_score((uint32_t)(last >> kIdxBits));
      p.jtie[o] = (int32_t)(kIdxMask - (last & kIdxMask));
      p.count[o] = (int32_t)((int64_t)sm.nabove[r] + take);
      if (p.mass) p.mass[o] = (float)(cum / Z);
    };

    // ---- sweeps 3+: level-1 score sub-bins, then composite-key digits, until
    // the crossing range is collected or parked
    for (int iter = 0;; ++iter) {
      const bool mine = state == ST_REFINE1 || state == ST_REFINE || state == ST_COLLECT ||
                        state == ST_LIST;
      if (g == 0) {
        sm.ncnt[r] = 0;
        sm.nabove[r] = 0;
      }
      bool any = bar_or(1, kEpi, mine);
      if (any && iter >= kMaxIter) {
        if (tid == 0) set_status(p.status, RTP_ERR_DEVICE_TIMEOUT, 14);
        any = false;
      }
      if (tid == 0) {  // tell the producer and the MMA issuer whether to sweep again
        *go = any ? 1 : 0;
        mbar_arrive(&sm.ctl);
      }
      if (!any) break;
      const int mode = state == ST_REFINE1  ? (int)MODE_SUB1
                       : state == ST_REFINE ? (int)MODE_DIGIT
                       : state == ST_COLLECT ? (int)MODE_COLLECT
                                             : (int)MODE_PARK;
      const int w = min(kDigit, kKeyBits - pbits);
      float lo = INFINITY, hi = -INFINITY;
      if (mine) refine_range(m, scale, margin, k0, k1, mode == MODE_SUB1 ? 0 : pbits, prefix, lo, hi);
      // rows gathering their range count the keys above it: past hi here, the
      // rest in drain_hits
      const bool counting = mine && mode >= MODE_COLLECT;
      const float hic = counting ? hi : INFINITY;
      // the prefilter |s - mid| <= half holds for every score in [lo, hi] (half
      // is rounded up); keys past hi that pass it are told apart in drain_hits
      float mid = 0.f, half = -1.f;
      if (mine) {
        mid = 0.5f * (lo + hi);
        half = __fmul_ru(__fsub_ru(hi, lo), 0.5f * (1.0f + 1.0f / 1048576.0f)) +
               fabsf(mid) * (1.0f / 4194304.0f) + 1e-30f;
        if (!(fabsf(mid) < INFINITY) || !(half < INFINITY)) {  // unbounded range
          mid = 0.f;
          half = INFINITY;
        }
      }
      const int wq = warp, row0 = (warp & 3) * 32;
      int qn = 0;  // entries in this warp's queue (warp-uniform)
      uint32_t n_above = 0u;
      auto drain = [&](int n) {
        drain_hits(sm, lists, wq, n, row0, g, m, scale, k0, k1, pbits, prefix, w, tk, mode, hic);
      };
      auto drain32 = [&]() {  // the queue's first 32 entries; the rest move down
        __syncwarp();
        drain(32);
        __syncwarp();
        if (lane + 32 < qn) {
          sm.t.q.s[wq][lane] = sm.t.q.s[wq][lane + 32];
          sm.t.q.jl[wq][lane] = sm.t.q.jl[wq][lane + 32];
        }
        __syncwarp();
        qn -= 32;
      };
      sweep(
          [&](int j0, float (&v)[kChunk]) {
            bool hit = false;
            const unsigned long long mid2 = f2_pack(mid, mid);
#pragma unroll
            for (int k = 0; k < kChunk / 2; ++k) {  // v - mid two lanes per instruction
              float d0, d1;
              f2_unpack(f2_sub(f2_pack(v[2 * k], v[2 * k + 1]), mid2), d0, d1);
              hit |= fabsf(d0) <= half;
              hit |= fabsf(d1) <= half;
              n_above += v[2 * k] > hic ? 1u : 0u;
              n_above += v[2 * k + 1] > hic ? 1u : 0u;
            }
            if (__ballot_sync(0xffffffffu, hit) == 0u) return;
            uint32_t hits = 0u;
#pragma unroll
            for (int i = 0; i < kChunk; ++i)
              hits |= (fabsf(__fsub_rn(v[i], mid)) <= half ? 1u : 0u) << i;
            // -0 -> +0 below: one composite key per score
            if (!__any_sync(0xffffffffu, (hits & (hits - 1u)) != 0u)) {
              // at most one hit per lane (the usual case): each hit lane writes
              // its key at its rank among the hit lanes (qn < 32 here, so the
              // queue holds them)
              const uint32_t bal = __ballot_sync(0xffffffffu, hits != 0u);
              if (hits != 0u) {
                const int i = __ffs(hits) - 1;
                const int pos = qn + __popc(bal & ((1u << lane) - 1u));
                sm.t.q.s[wq][pos] = pick16(v, i) + 0.0f;
                sm.t.q.jl[wq][pos] = (uint32_t)(j0 + i) | ((uint32_t)lane << 21);
              }
              qn += __popc(bal);
              if (qn >= 32) drain32();
              return;
            }
            const int nh = __popc(hits);
            int incl = nh;  // inclusive prefix sum of the lanes' hit counts
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
              const int t = __shfl_up_sync(0xffffffffu, incl, o);
              if (lane >= o) incl += t;
            }
            const int total = __shfl_sync(0xffffffffu, incl, 31);
            if (qn + total <= kQueue) {  // every lane writes its hits at once
              int pos = qn + incl - nh;
#pragma unroll
              for (int i = 0; i < kChunk; ++i)
                if ((hits >> i) & 1u) {
                  sm.t.q.s[wq][pos] = v[i] + 0.0f;
                  sm.t.q.jl[wq][pos] = (uint32_t)(j0 + i) | ((uint32_t)lane << 21);
                  ++pos;
                }
              qn += total;
              while (qn >= 32) drain32();
            } else {  // a dense chunk: one key position at a time
              const uint32_t lt = (1u << lane) - 1u;
#pragma unroll
              for (int i = 0; i < kChunk; ++i) {
                const bool h = (hits >> i) & 1u;
                const uint32_t bal = __ballot_sync(0xffffffffu, h);
                if (bal == 0u) continue;
                if (h) {
                  const int pos = qn + __popc(bal & lt);
                  sm.t.q.s[wq][pos] = v[i] + 0.0f;
                  sm.t.q.jl[wq][pos] = (uint32_t)(j0 + i) | ((uint32_t)lane << 21);
                }
                qn += __popc(bal);
                if (qn >= 32) drain32();
              }
            }
          },
          true, mine && mode <= MODE_DIGIT);
      if (qn > 0) {  // the last partial batch
        __syncwarp();
        drain(qn);
      }
      if (counting) atomicAdd(&sm.nabove[r], (int)n_above);
      ebar();
      if (g == 0 && mine && mode <= MODE_DIGIT) flush_row(sm, r);
      ebar();
      // a row that parked its range this sweep (a row that turns to ST_LIST
      // below parks in the next sweep)
      const bool lst = mine && mode == MODE_PARK;
      const int nl = lst ? min(sm.ncnt[r], kListCap) : 0;
      auto fd = [&](int) { return fk; };
      if (mine && mode == MODE_COLLECT) {
        if (g == 0) finish_row();
        state = ST_DONE;
      } else if (mine && mode == MODE_SUB1) {
        unsigned long long wsel = 0ull;
        const int b1 = crossing(sm, r, kNB, T, false, fd, base, inner, wsel);
        if (b1 < 0) set_status(p.status, RTP_ERR_DEVICE_TIMEOUT, 17);
        k1 = max(b1, 0);
        const float s32 = scale * (float)kNB;
        umin = fmaxf(2097152.0f * expf(-(float)(k1 + 1) / s32) * (1.0f - 1.0f / 1024.0f) - 1.0f,
                     1.0f);
        n_cur = bound(wsel);
        range_prefix(m - (float)(kNB * k0 + k1 + 1) / s32, m - (float)(kNB * k0 + k1) / s32,
                     margin, pbits, prefix);
        state = next_state(n_cur, false);
      } else if (mine && mode == MODE_DIGIT) {
        unsigned long long wsel = 0ull;
        const int bsel = crossing(sm, r, 1 << w, T, false, fd, base, inner, wsel);
        if (bsel < 0) set_status(p.status, RTP_ERR_DEVICE_TIMEOUT, 18);
        prefix = (prefix << w) | (unsigned long long)((1 << w) - 1 - max(bsel, 0));
        pbits += w;
        n_cur = bound(wsel);
        state = next_state(n_cur, false);
      }
      ebar();
      if (g == 0 && (state == ST_REFINE || (state == ST_LIST && !lst))) clear_row(sm, r);
      // rows with a parked list: the remaining digit levels run over the list, a
      // warp per row at a time (lanes read consecutive entries).  Each level keeps
      // the entries of the current prefix in place and in order, and counts the
      // ones above it; the row's own threads keep the selection state and publish
      // what the warps read in shared memory
      if (bar_or(1, kEpi, lst)) {
        auto& ls = sm.t.ls;
        const uint32_t lt = (1u << lane) - 1u;
        if (g == 0) {
          ls.n[r] = lst ? nl : 0;
          ls.m[r] = m;
          ls.tk[r] = tk;
        }
        for (;;) {
          const bool need = lst && n_cur > (unsigned long long)kCap && pbits < kKeyBits;
          if (g == 0) {
            ls.need[r] = need ? 1 : 0;
            ls.prefix[r] = prefix;
            ls.pbits[r] = pbits;
          }
          if (!bar_or(1, kEpi, need)) break;
          for (int rr = warp; rr < kBM; rr += kEpi / 32) {
            if (!ls.need[rr]) continue;
            const unsigned long long pfx = ls.prefix[rr];
            const int pb = ls.pbits[rr], wl = min(kDigit, kKeyBits - pb), n = ls.n[rr];
            const float rm = ls.m[rr], rtk = ls.tk[rr];
            unsigned long long* const L = lists + (size_t)rr * kListCap;
            int kept = 0, above = 0;
            // kListBatch entries per lane are loaded before any is written back:
            // the compacted entries land at or below the batch's own positions,
            // never on an entry still to be loaded
            for (int kb0 = 0; kb0 < n; kb0 += 32 * kListBatch) {
              unsigned long long cb[kListBatch];
#pragma unroll
              for (int u = 0; u < kListBatch; ++u) {
                const int k = kb0 + 32 * u + lane;
                cb[u] = k < n ? __ldcg(L + k) : 0ull;
              }
#pragma unroll
              for (int u = 0; u < kListBatch; ++u) {
                const int k0 = kb0 + 32 * u;
                if (k0 >= n) break;
                if (k0 > 0 && k0 % kListFlush == 0) {  // only this warp adds to row rr
                  __syncwarp();
                  if (lane < kNB) {
                    sm.u.hw[lane][rr] +=
                        (unsigned long long)sm.wacc[0][lane][rr] + sm.wacc[1][lane][rr];
                    sm.wacc[0][lane][rr] = 0u;
                    sm.wacc[1][lane][rr] = 0u;
                  }
                  __syncwarp();
                }
                const int k = k0 + lane;
                const unsigned long long ck = cb[u];
                const unsigned long long px = pb > 0 ? (ck >> (kKeyBits - pb)) : 0ull;
                const bool in = (k < n) & (px == pfx);
                above += ((k < n) & (px > pfx)) ? 1 : 0;
                const uint32_t ball = __ballot_sync(0xffffffffu, in);
                if (in) {
                  L[kept + __popc(ball & lt)] = ck;
                  const int digit = (int)((ck >> (kKeyBits - pb - wl)) & ((1ull << wl) - 1));
                  // even and odd entries in separate copies: <= 2032 keys each
                  // between flushes
                  atomicAdd(&sm.wacc[lane & 1][(1 << wl) - 1 - digit][rr],
                            fixed_u(__fmul_rn(rel_w(key_score((uint32_t)(ck >> kIdxBits)), rm),
                                              rtk)));
                }
                kept += __popc(ball);
              }
            }
            above = __reduce_add_sync(0xffffffffu, above);
            if (lane == 0) {
              ls.n[rr] = kept;
              sm.nabove[rr] += above;
            }
          }
          ebar();
          if (need && g == 0) flush_row(sm, r);
          ebar();
          if (need) {
            unsigned long long wsel = 0ull;
            const int wl = min(kDigit, kKeyBits - pbits);
            const int bsel = crossing(sm, r, 1 << wl, T, false, fd, base, inner, wsel);
            if (bsel < 0) set_status(p.status, RTP_ERR_DEVICE_TIMEOUT, 19);
            prefix = (prefix << wl) | (unsigned long long)((1 << wl) - 1 - max(bsel, 0));
            pbits += wl;
            n_cur = bound(wsel);
          }
          ebar();
          if (need && g == 0) clear_row(sm, r);
        }
        // the final range's keys become the row's candidates
        if (g == 0) {
          ls.need[r] = lst ? 1 : 0;
          ls.prefix[r] = prefix;
          ls.pbits[r] = pbits;
          sm.ncnt[r] = 0;
        }
        ebar();
        for (int rr = warp; rr < kBM; rr += kEpi / 32) {
          if (!ls.need[rr]) continue;
          const unsigned long long pfx = ls.prefix[rr];
          const int pb = ls.pbits[rr], n = ls.n[rr];
          const unsigned long long* const L = lists + (size_t)rr * kListCap;
          int above = 0;
          for (int kb0 = 0; kb0 < n; kb0 += 32 * kListBatch) {
            unsigned long long cb[kListBatch];
#pragma unroll
            for (int u = 0; u < kListBatch; ++u) {
              const int k = kb0 + 32 * u + lane;
              cb[u] = k < n ? __ldcg(L + k) : 0ull;
            }
#pragma unroll
            for (int u = 0; u < kListBatch; ++u) {
              if (kb0 + 32 * u + lane >= n) break;
              const unsigned long long ck = cb[u];
              const unsigned long long px = pb > 0 ? (ck >> (kKeyBits - pb)) : 0ull;
              if (px == pfx) {
                const int slot_c = atomicAdd(&sm.ncnt[rr], 1);
                if (slot_c < kCap) sm.u.cand[slot_c][rr] = ck;
              } else if (px > pfx) {
                ++above;
              }
            }
          }
          above = __reduce_add_sync(0xffffffffu, above);
          if (lane == 0) sm.nabove[rr] += above;
        }
      }
      ebar();
      if (lst) {
        if (g == 0) finish_row();
        state = ST_DONE;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (tid == 0 && sm.slot >= 0) {  // the list slot is free again
    __threadfence();
    atomicAnd(&p.slot_mask[sm.slot >> 1], ~(1u << (sm.slot & 1)));
  }
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * kBN);
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

namespace rtp {
// Workspace of rtp_topp_select: the status word, one slot-occupancy word per SM
// and two candidate-list slots per SM of kBM x kListCap composite keys.
SelectWs select_ws_layout() {
  SelectWs w{};
  int dev = 0, n_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      n_sm <= 0) {
    cudaGetLastError();
    return w;  // total 0: lists off
  }
  w.n_sm = n_sm;
  w.mask = kStatusBytes;
  w.lists = w.mask + (((size_t)n_sm * 4 + 255) / 256) * 256;
  w.total = w.lists + (size_t)2 * n_sm * kBM * kListCap * 8;
  return w;
}
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
  const SelectWs wl = select_ws_layout();
  if (p >= 1.f) {
    TraceScope tr("topp_all", s);
    topp_all_kernel<<<592, 256, 0, s>>>(hm.n_ret, shape->Lq, shape->q_pos0, shape->B, thr,
                                        jtie, count, mass);
    return check_cuda(cudaGetLastError());
  }
  if ((st = check_view(q16, hm.n_ret, kR, true)) != RTP_OK) return st;
  if ((st = check_view(k16, hm.H_k16, kR, true)) != RTP_OK) return st;
  SelParams prm;
  // with a full-size workspace, rows may park dense crossing bins in lists
  const bool with_lists = wl.total > 0 && ws_bytes >= wl.total;
  prm.lists = with_lists ? reinterpret_cast<unsigned long long*>(static_cast<char*>(ws) + wl.lists)
                         : nullptr;
  prm.slot_mask = with_lists ? reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + wl.mask)
                             : nullptr;
  prm.n_sm = wl.n_sm;
  prm.Lq = shape->Lq;
  prm.q_pos0 = shape->q_pos0;
  prm.n_ret = hm.n_ret;
  prm.p = p;
  prm.thr = thr;
  prm.jtie = jtie;
  prm.count = count;
  prm.mass = mass;
  prm.status = static_cast<DevStatus*>(ws);
  for (int i = 0; i < hm.n_ret; ++i) prm.k16_slot[i] = hm.ret_k16[i];
  // q16 / k16 as 4-D tensors {16, slots, rows, batch}; 128-row boxes of one slot,
  // 32-byte swizzled (the canonical K-major operand layout of the MMA)
  prm.batch_coord_q = (q16.stride_b != 0 || shape->B == 1) ? 1 : 0;
  prm.batch_coord_k = (k16.stride_b != 0 || shape->B == 1) ? 1 : 0;
  CUtensorMap qmap, kmap;
  {
    const uint64_t sl = (uint64_t)q16.stride_l * 2;
    const uint64_t sb = prm.batch_coord_q && q16.stride_b != 0 ? (uint64_t)q16.stride_b * 2
                                                               : sl * (uint64_t)shape->Lq;
    const uint64_t dims[4] = {16, (uint64_t)hm.n_ret, (uint64_t)shape->Lq,
                              prm.batch_coord_q ? (uint64_t)shape->B : 1u};
    const uint64_t strides[3] = {32, sl, sb};
    const uint32_t box[4] = {16, 1, (uint32_t)kBM, 1};
    if (!tma_encode_bf16(&qmap, q16.ptr, 4, dims, strides, box, 32)) return RTP_ERR_CUDA;
  }
  {
    const uint64_t sl = (uint64_t)k16.stride_l * 2;
    const uint64_t sb = prm.batch_coord_k && k16.stride_b != 0 ? (uint64_t)k16.stride_b * 2
                                                               : sl * (uint64_t)shape->Lk;
    const uint64_t dims[4] = {16, (uint64_t)hm.H_k16, (uint64_t)shape->Lk,
                              prm.batch_coord_k ? (uint64_t)shape->B : 1u};
    const uint64_t strides[3] = {32, sl, sb};
    const uint32_t box[4] = {16, 1, (uint32_t)kBN, 1};
    if (!tma_encode_bf16(&kmap, k16.ptr, 4, dims, strides, box, 32)) return RTP_ERR_CUDA;
  }
  const size_t smem = sizeof(SelSmem) + 1024;
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
  topp_select_kernel<<<grid, kThreads, smem, s>>>(qmap, kmap, prm);
  return check_cuda(cudaGetLastError());
}
