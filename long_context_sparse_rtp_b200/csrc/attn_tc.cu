// attn_tc.cu -- causal prefill attention tiles on the 5th-generation tensor
// cores, for the three head kinds:
//
//   DENSE  every key j <= P (baseline);
//   LOCAL  keys j <= P with j < n_sink or j > P - window ("Local Head Attention
//          Pattern" of the paper-graph-ui summary of arXiv 2605.16928); key
//          tiles outside the sinks and the window are never visited;
//   SPARSE keys j <= P kept by the row's top-p descriptor (thr, jtie) ("Dynamic
//          Top-p Selection Mechanism"): each tile's 16-dim indexer scores are
//          recomputed by the same tcgen05 MMA shape and operand placement the
//          selection used (128 query rows x 128 keys, K = 16), so the kept set
//          is reproduced bit for bit.
//
// One CTA = 128 query rows of one head, 128-key tiles.  Warp 8 loads Q once and
// K/V (and K16) tiles into a 2-stage ring with TMA (128-byte swizzle); warp 9
// issues S = Q K^T (8 MMAs, K = 16 each) into one of two TMEM score buffers and
// O += P V into a TMEM accumulator; warps 0-7 hold two threads per query row
// (64 keys and 64 output dimensions each): read the scores with tcgen05.ld,
// mask, share the tile max with the partner thread, online softmax in the log2
// domain, write P (bf16, two per column) over the scores in TMEM, where the PV
// MMA reads it as its A operand.  The running max is only
// moved (and O rescaled in TMEM) when it grows by more than 2^8, so most tiles
// need no rescale.  P is rounded to bf16 once for the PV MMA; the normaliser
// sums the fp32 values.
#include <cuda.h>

#include "rtp_host.h"
#include "tcgen05.cuh"
#include "tma.cuh"

namespace rtp {
namespace {

constexpr int kBM = 128;                  // query rows per CTA (TMEM lanes)
constexpr int kBN = 128;                  // keys per tile
constexpr int kStages = 2;                // K/V ring
constexpr int kHalf = 128 * 128;          // one 64-column half of a 128 x 128 bf16 tile: 16 KB
constexpr int kTile = 2 * kHalf;          // 32 KB
constexpr int kSoftmax = 256;            // softmax threads: two per query row
constexpr int kProdWarp = kSoftmax / 32, kMmaWarp = kProdWarp + 1;
constexpr int kThreads = kSoftmax + 64;
constexpr float kRescale = 8.f;           // move the max when it grows by > 2^8
constexpr uint32_t kIdescQK = idesc_bf16_f32(kBM, kBN);
constexpr uint32_t kIdescPV = idesc_bf16_f32(kBM, kD) | (1u << 16);  // V is MN-major

enum { MODE_DENSE = 0, MODE_LOCAL = 1, MODE_SPARSE = 2 };

struct AttnParams {
  uint16_t* o; int64_t o_sb, o_sl;
  float* lse;                // [B][H][Lq] or null
  DevStatus* status;
  const float* thr;          // [B][n_ret][Lq]
  const int32_t* jtie;
  int Lq, Lk, H, G, n_ret;
  int64_t q_pos0;
  int window, n_sink;
  int bq, bk;                // batch coordinate multipliers (0 when a tensor is shared)
  float scale_log2;          // softmax_scale * log2(e)
  int16_t head[kMaxHeads];   // launch head index -> query head
  int16_t slot[kMaxHeads];   // launch head index -> retrieval slot (SPARSE)
  int16_t k16slot[kMaxHeads];// launch head index -> k16 slot (SPARSE)
};

struct TcSmem {                      // placed on a 1024-byte boundary
  uint8_t q[kTile];                  // [2 halves of 64 dims][128 rows][128 B]
  uint8_t k[kStages][kTile];
  uint8_t v[kStages][kTile];         // rows = keys, 2 halves of 64 dims (MN-major B)
  uint8_t q16[kBM * kR * 2];         // 32-byte rows, 32-byte swizzle
  uint8_t k16[kStages][kBN * kR * 2];
  // per-tile barriers with several arriving warps come in pairs by tile parity:
  // a warp may run one tile ahead of another, never two
  uint64_t q_full, kv_full[kStages], kv_empty[kStages], s_full[2], s_empty[2], s16_empty[2],
      p_full[2], o_done[2];
  float tmax[2][2][kBM];             // [tile parity][column half][row]: partial tile maxima
  float lpart[2][kBM];               // [column half][row]: partial row sums
  uint32_t tmem_base;
  int gave_up;
};

// The key-tile schedule of a row block: LOCAL visits the sink tiles, then the
// window tiles; the other modes every tile up to the diagonal.
struct Sched {
  int n, sink_end, win_begin;
  __device__ __forceinline__ int tile(int it) const {
    return it < sink_end ? it : win_begin + (it - sink_end);
  }
};

// The largest float below t (t = -inf stays -inf; no denormal flushing, so the
// float below 0 is the negative least denormal and s > it iff s >= 0).
__device__ __forceinline__ float float_below(float t) {
  if (!(t > -INFINITY)) return t;
  if (t == 0.f) return __uint_as_float(0x80000001u);
  const uint32_t u = __float_as_uint(t);
  return __uint_as_float(t > 0.f ? u - 1u : u + 1u);
}

__device__ __forceinline__ float ex2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}
// The row-sum slots of a half tile (pairs e of keys 2e, 2e + 1 go to slot e % 4,
// even keys in the low lane, odd in the high), folded in a fixed order.
__device__ __forceinline__ float fold_sums(const unsigned long long (&ls)[4]) {
  float a[4], b[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) f2_unpack(ls[k], a[k], b[k]);
  return ((a[0] + b[0]) + (a[1] + b[1])) + ((a[2] + b[2]) + (a[3] + b[3]));
}

template <int MODE>
__device__ __forceinline__ Sched make_sched(const AttnParams& p, int64_t P0, int64_t Plast) {
  Sched s;
  const int t_end = (int)(Plast / kBN);  // inclusive
  if (MODE == MODE_LOCAL) {
    int sink_end = (p.n_sink + kBN - 1) / kBN;
    const int64_t wlo = P0 - p.window + 1;  // lowest window key of the block's first row
    int win_begin = (int)((wlo > 0 ? wlo : 0) / kBN);
    if (win_begin < sink_end) win_begin = sink_end;
    sink_end = min(sink_end, t_end + 1);
    s.sink_end = sink_end;
    s.win_begin = win_begin;
    s.n = sink_end + max(0, t_end - win_begin + 1);
  } else {
    s.sink_end = t_end + 1;
    s.win_begin = t_end + 1;
    s.n = t_end + 1;
  }
  return s;
}

// K-major operand descriptor: K step kk (16 elements) of a 128 x 128 tile.
__device__ __forceinline__ uint64_t kdesc(const uint8_t* tile, int kk) {
  return sdesc_sw128(smem_u32(tile) + (uint32_t)((kk >> 2) * kHalf + (kk & 3) * 32), 16, 1024);
}
// MN-major V descriptor: K step kk (16 keys = 2 KB of rows), 64-dim halves kHalf apart.
__device__ __forceinline__ uint64_t vdesc(const uint8_t* tile, int kk) {
  return sdesc_sw128(smem_u32(tile) + (uint32_t)(kk * 2048), kHalf, 1024);
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap qmap,
                   const __grid_constant__ CUtensorMap kmap,
                   const __grid_constant__ CUtensorMap vmap,
                   const __grid_constant__ CUtensorMap q16map,
                   const __grid_constant__ CUtensorMap k16map, const AttnParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  TcSmem& sm = *reinterpret_cast<TcSmem*>(smem_raw +
                                          ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int hidx = blockIdx.y;
  const int h = p.head[hidx];
  const int kvh = h / p.G;
  const int b = blockIdx.z;
  const int rb = gridDim.x - 1 - blockIdx.x;  // heavy (late) row blocks first
  const int m0 = rb * kBM;
  const int nrows = min(kBM, p.Lq - m0);
  const int64_t P0 = p.q_pos0 + m0;
  const int64_t Plast = P0 + nrows - 1;
  const Sched sch = make_sched<MODE>(p, P0, Plast);
  const bool sparse = MODE == MODE_SPARSE;

  if (tid == 0) {
    mbar_init(&sm.q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.s_full[i], 1);
      mbar_init(&sm.s_empty[i], 1);  // committed once the PV MMA reading P from it is done
      mbar_init(&sm.o_done[i], 1);   // PV MMAs of tiles with this parity
      mbar_init(&sm.s16_empty[i], kSoftmax / 32);
      mbar_init(&sm.p_full[i], kSoftmax / 32);
    }
    sm.gave_up = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const uint32_t t_s = tmem, t_o = tmem + 256, t_s16 = tmem + 384;
  volatile int* gave_up = &sm.gave_up;

  if (warp == kProdWarp) {  // ---------------------------------------- TMA producer
    if (lane == 0) {
      bool ok = true;
      const uint32_t qbytes = kTile + (sparse ? kBM * kR * 2 : 0);
      const uint32_t kvbytes = 2 * kTile + (sparse ? kBN * kR * 2 : 0);
      mbar_arrive_expect_tx(&sm.q_full, qbytes);
      tma_load_4d(sm.q, &qmap, 0, h, m0, b * p.bq, &sm.q_full);
      tma_load_4d(sm.q + kHalf, &qmap, 64, h, m0, b * p.bq, &sm.q_full);
      if (sparse) tma_load_4d(sm.q16, &q16map, 0, p.slot[hidx], m0, b * p.bq, &sm.q_full);
      int n_issued = 0;
      for (int it = 0; it < sch.n; ++it) {
        const int st = it & 1;
        if (!mbar_wait(&sm.kv_empty[st], ((uint32_t)(it >> 1) & 1u) ^ 1u, gave_up)) {
          ok = false;
          break;
        }
        const int j0 = sch.tile(it) * kBN;
        mbar_arrive_expect_tx(&sm.kv_full[st], kvbytes);
        tma_load_4d(sm.k[st], &kmap, 0, kvh, j0, b * p.bk, &sm.kv_full[st]);
        tma_load_4d(sm.k[st] + kHalf, &kmap, 64, kvh, j0, b * p.bk, &sm.kv_full[st]);
        tma_load_4d(sm.v[st], &vmap, 0, kvh, j0, b * p.bk, &sm.kv_full[st]);
        tma_load_4d(sm.v[st] + kHalf, &vmap, 64, kvh, j0, b * p.bk, &sm.kv_full[st]);
        if (sparse)
          tma_load_4d(sm.k16[st], &k16map, 0, p.k16slot[hidx], j0, b * p.bk, &sm.kv_full[st]);
        ++n_issued;
      }
      if (!ok) set_status(p.status, RTP_ERR_DEVICE_TIMEOUT, 41);
      for (int k = max(0, n_issued - kStages); k < n_issued; ++k)
        mbar_wait_drain(&sm.kv_full[k & 1], (uint32_t)(k >> 1) & 1u);
      mbar_wait_drain(&sm.q_full, 0u);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {  // ---------------------------------- MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(&sm.q_full, 0u, gave_up);
      uint32_t n_pv = 0;
      // O += P V for tile `it`, P read from TMEM (its score buffer); the K/V stage
      // and the score buffer are released when the MMAs are done
      auto pv = [&](int it) {
        if (!mbar_wait(&sm.p_full[it & 1], (uint32_t)(it >> 1) & 1u, gave_up)) return false;
        tc_fence_after();
        const int st = it & 1, sb = it & 1;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ts(t_o, t_s + (uint32_t)(sb * kBN + kk * 8), vdesc(sm.v[st], kk), kIdescPV,
                      it > 0 || kk > 0);
        mma_commit(&sm.o_done[it & 1]);
        mma_commit(&sm.s_empty[sb]);
        mma_commit(&sm.kv_empty[st]);
        ++n_pv;
        return true;
      };
      for (int it = 0; ok && it < sch.n; ++it) {
        const int st = it & 1, sb = it & 1;
        // S16 of tile it-1 must have been read before S16 of tile it overwrites it
        if (!mbar_wait(&sm.kv_full[st], (uint32_t)(it >> 1) & 1u, gave_up) ||
            !mbar_wait(&sm.s_empty[sb], ((uint32_t)(it >> 1) & 1u) ^ 1u, gave_up) ||
            (sparse && it > 0 &&
             !mbar_wait(&sm.s16_empty[(it - 1) & 1], (uint32_t)((it - 1) >> 1) & 1u, gave_up))) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ss(t_s + (uint32_t)(sb * kBN), kdesc(sm.q, kk), kdesc(sm.k[st], kk),
                      kIdescQK, kk > 0);
        if (sparse)
          mma_bf16_ss(t_s16, sdesc_k_sw32(smem_u32(sm.q16), 256),
                      sdesc_k_sw32(smem_u32(sm.k16[st]), 256), kIdescQK, false);
        mma_commit(&sm.s_full[sb]);
        if (it > 0 && !pv(it - 1)) ok = false;  // S(it) overlaps the softmax of tile it-1
      }
      if (ok && sch.n > 0 && !pv(sch.n - 1)) ok = false;
      if (!ok) set_status(p.status, RTP_ERR_DEVICE_TIMEOUT, 42);
      if (n_pv > 0) mbar_wait_drain(&sm.o_done[(n_pv - 1) & 1u], ((n_pv - 1) >> 1) & 1u);
    }
    __syncwarp();
  } else {  // ------------------------------- softmax: two threads per query row
    // thread (r, g): TMEM lane r, key columns 64 g .. 64 g + 63 of each tile, output
    // dimensions 64 g .. 64 g + 63.  Warps w and w + 4 hold the same rows and
    // exchange their tile maxima through shared memory (pair barrier 1 + w % 4).
    const int r = tid & (kBM - 1), g = tid >> 7;
    const bool valid = r < nrows;
    const int64_t P = P0 + r;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const int pair_bar = 1 + (warp & 3);
    float thr = INFINITY;
    int64_t jt = -1;
    if (sparse && valid) {
      const int64_t ob = ((int64_t)b * p.n_ret + p.slot[hidx]) * p.Lq + m0 + r;
      thr = p.thr[ob];
      jt = p.jtie[ob];
    }
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int it = 0; it < sch.n; ++it) {
      const int sb = it & 1;
      const int64_t j0 = (int64_t)sch.tile(it) * kBN + g * 64;  // this thread's first key
      ok = ok && mbar_wait_warp(&sm.s_full[sb], (uint32_t)(it >> 1) & 1u, gave_up);
      tc_fence_after();
      const uint32_t col = (uint32_t)(sb * kBN + g * 64);
      // the thread's 64 scores, masked and scaled into the log2 domain
      float x[64];
      if (sparse) {
        // the indexer predicate: s16 > t, or s16 == t and j <= jtie; causal j <= P.
        // One compare per key against te = t, or the float below t where the tie
        // index lies past these keys (every tie kept); keys holding a lane's tie
        // index or the diagonal take one more select each
        auto clamp_off = [](int64_t d) { return (int)(d < -1 ? -1 : (d > 63 ? 63 : d)); };
        const int ptl = clamp_off(P - j0), jtl = clamp_off(jt - j0);
        const float te = !ok ? INFINITY : (jtl == 63 ? float_below(thr) : thr);
        const bool mixed = __any_sync(0xffffffffu, (jtl >= 0) & (jtl < 63));
        const bool diag = __any_sync(0xffffffffu, ptl < 63);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t r16[32], rs[32];
          if (ok) {
            tmem_ld32_nowait(t_s16 + lane_off + (uint32_t)(g * 64 + c * 32), r16);
            tmem_ld32_nowait(t_s + lane_off + col + (uint32_t)(c * 32), rs);
            tmem_wait_ld();
          }
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            reg_fence(r16[i]);
            reg_fence(rs[i]);
            x[c * 32 + i] = __uint_as_float(r16[i]) > te ? __uint_as_float(rs[i]) : -INFINITY;
          }
          if (mixed) {  // ties up to the tie index (-0 and +0 compare equal)
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const bool tie = ok & (__uint_as_float(r16[i]) == thr) & (c * 32 + i <= jtl);
              x[c * 32 + i] = tie ? __uint_as_float(rs[i]) : x[c * 32 + i];
            }
          }
        }
        if (diag) {
#pragma unroll
          for (int i = 0; i < 64; ++i) x[i] = i <= ptl ? x[i] : -INFINITY;
        }
        tc_fence_before();  // S16 is in registers: the MMA may reuse its buffer
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.s16_empty[it & 1]);
      } else {
        if (ok) {
          float a[32], c2[32];
          tmem_ld32(t_s + lane_off + col, a);
          tmem_ld32(t_s + lane_off + col + 32u, c2);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            x[i] = a[i];
            x[32 + i] = c2[i];
          }
        }
        bool full = false;
        if (MODE == MODE_DENSE) full = j0 + 63 <= P;
        if (MODE == MODE_LOCAL) full = j0 + 63 <= P && (j0 > P - p.window || j0 + 63 < p.n_sink);
        if (!(full && ok)) {
#pragma unroll
          for (int i = 0; i < 64; ++i) {
            const int64_t j = j0 + i;
            bool kp;
            if (MODE == MODE_DENSE) kp = j <= P;
            else kp = (j <= P) & ((j < p.n_sink) | (j > P - p.window));
            x[i] = (ok & kp) ? x[i] : -INFINITY;
          }
        }
      }
      float tm[8];  // the thread's max as a tree (independent chains)
#pragma unroll
      for (int e = 0; e < 8; ++e) tm[e] = x[e];
#pragma unroll
      for (int i = 8; i < 64; i += 2) tm[(i >> 1) & 7] = max3f(tm[(i >> 1) & 7], x[i], x[i + 1]);
      // in the log2 domain (scale > 0 keeps the order; -inf stays -inf)
      float tmax = fmaxf(fmaxf(fmaxf(tm[0], tm[1]), fmaxf(tm[2], tm[3])),
                         fmaxf(fmaxf(tm[4], tm[5]), fmaxf(tm[6], tm[7]))) *
                   p.scale_log2;
      // the row's tile max from the partner thread (parity-paired slots)
      sm.tmax[it & 1][g][r] = tmax;
      named_bar(pair_bar, 64);
      tmax = fmaxf(tmax, sm.tmax[it & 1][g ^ 1][r]);
      const float m_new = fmaxf(m_used, tmax);
      const bool first = m_used == -INFINITY && m_new > -INFINITY;  // O and l are still 0
      const bool move = m_used > -INFINITY && m_new > m_used + kRescale;
      float alpha = 1.f;
      if (first) m_used = m_new;
      if (move) {
        alpha = exp2f(m_used - m_new);
        m_used = m_new;
        l *= alpha;
      }
      // O is rescaled (rarely) once the previous tile's PV MMA is done: this
      // thread's 64 dimensions
      if (it > 0 && __any_sync(0xffffffffu, move)) {
        ok = ok && mbar_wait_warp(&sm.o_done[(it - 1) & 1], (uint32_t)((it - 1) >> 1) & 1u,
                                  gave_up);
        tc_fence_after();
        if (ok) {
#pragma unroll 1
          for (int c = 0; c < 2; ++c) {
            float o[32];
            tmem_ld32(t_o + lane_off + (uint32_t)(g * 64 + c * 32), o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tmem_st32(t_o + lane_off + (uint32_t)(g * 64 + c * 32), o);
          }
        }
      }
      // P = 2^(x - m) rounded to bf16 once, packed two per column over the scores:
      // keys 64 g + 2e, 64 g + 2e + 1 go to column 32 g + e of the tile's buffer
      const float msafe = m_used == -INFINITY ? 0.f : m_used;  // masked keys: 2^-inf = 0
      unsigned long long lsum[4] = {0ull, 0ull, 0ull, 0ull};  // (+0, +0) pairs
      {
        const unsigned long long cc = f2_pack(p.scale_log2, p.scale_log2);
        const unsigned long long mm = f2_pack(-msafe, -msafe);
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          float x0, x1;
          f2_unpack(f2_fma(f2_pack(x[2 * e], x[2 * e + 1]), cc, mm), x0, x1);
          const float p0 = ex2_ftz(x0), p1 = ex2_ftz(x1);
          pk[e] = pack_bf16x2(p0, p1);
          lsum[e & 3] = f2_add(lsum[e & 3], f2_pack(p0, p1));
        }
        if (ok) tmem_st32u(t_s + lane_off + (uint32_t)(sb * kBN + g * 32), pk);
      }
      tmem_wait_st();
      l += fold_sums(lsum);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.p_full[it & 1]);
    }
    // ---- epilogue: O / l from TMEM, bf16 rows to global (64 dimensions each)
    sm.lpart[g][r] = l;
    named_bar(pair_bar, 64);
    const float lrow = l + sm.lpart[g ^ 1][r];
    if (sch.n > 0)
      ok = ok && mbar_wait_warp(&sm.o_done[(sch.n - 1) & 1], (uint32_t)((sch.n - 1) >> 1) & 1u,
                                gave_up);
    tc_fence_after();
    const float inv = lrow > 0.f ? 1.f / lrow : 0.f;
    uint16_t* orow = p.o + b * p.o_sb + (int64_t)(m0 + r) * p.o_sl + (int64_t)h * kD + g * 64;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      float o[32];
      if (sch.n > 0) {
        tmem_ld32(t_o + lane_off + (uint32_t)(g * 64 + c * 32), o);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = 0.f;
      }
      if (valid) {
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          uint4 w;
          w.x = pack_bf16x2(o[q4 * 8 + 0] * inv, o[q4 * 8 + 1] * inv);
          w.y = pack_bf16x2(o[q4 * 8 + 2] * inv, o[q4 * 8 + 3] * inv);
          w.z = pack_bf16x2(o[q4 * 8 + 4] * inv, o[q4 * 8 + 5] * inv);
          w.w = pack_bf16x2(o[q4 * 8 + 6] * inv, o[q4 * 8 + 7] * inv);
          *reinterpret_cast<uint4*>(orow + c * 32 + q4 * 8) = w;
        }
      }
    }
    if (g == 0 && valid && p.lse != nullptr)
      p.lse[((int64_t)b * p.H + h) * p.Lq + m0 + r] =
          lrow > 0.f ? (m_used + log2f(lrow)) * kLn2 : -INFINITY;
    if (!ok && r == 0 && g == 0) set_status(p.status, RTP_ERR_DEVICE_TIMEOUT, 43);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// DENSE and LOCAL on two query tiles per CTA.
//
// One CTA = 256 query rows of one head (two 128-row tiles A and B) and one pass
// over the union of their key tiles.  TMEM holds, per query tile, a 128-column
// score buffer (P is written over it) and a 128-column O accumulator.  Warp 9
// issues, per key tile t: PV_A(t), S_A(t+1), PV_B(t), S_B(t+1), so the softmax
// of one tile runs while the tensor cores work on the other's.  Warps 0-3 hold
// the rows of tile A, warps 4-7 those of B: one thread per query row, all 128
// keys of a key tile (read from TMEM twice: the row max, then P), no exchange
// with another thread.  Warp 8 loads both Q tiles once and K/V tiles into a
// 2-stage ring with TMA.  Same arithmetic as the single-tile kernel: scores
// scaled into the log2 domain, the running max moved (and O rescaled) only when
// it grows by more than 2^8, P rounded to bf16 once for the MMA and summed in fp32,
// in the single-tile kernel's order (the two give the same bits).
constexpr int kPQ = 2;                     // query tiles per CTA
constexpr int kPRows = kPQ * kBM;          // 256

struct PpSmem {                            // placed on a 1024-byte boundary
  uint8_t q[kPQ][kTile];
  uint8_t k[kStages][kTile];
  uint8_t v[kStages][kTile];
  // each completes once per key tile: s_full[q] (the S MMAs of tile q),
  // p_full[q] (tile q's four softmax warps wrote P), pv_done[q] (its PV MMAs)
  uint64_t q_full, kv_full[kStages], kv_empty[kStages], s_full[kPQ], p_full[kPQ], pv_done[kPQ];
  uint32_t tmem_base;
  int gave_up;
};

// A key tile of the two-tile kernel that some row of the warp attends to only in
// part: the scores of keys outside the rule (key i kept iff i <= dp and (i < ds
// or i > dw)) become -inf in this thread's TMEM lane (columns ts .. ts + 127),
// 32 columns at a time, skipping chunks no row of the warp masks.
__device__ __forceinline__ void pp_mask(uint32_t ts, int dp, int ds, int dw) {
#pragma unroll 1
  for (int w = 0; w < 4; ++w) {
    const int k0 = 32 * w;
    const bool whole = k0 + 31 <= dp && (ds >= k0 + 32 || dw < k0);
    if (__all_sync(0xffffffffu, whole)) continue;
    uint32_t ra[32];
    tmem_ld32_nowait(ts + (uint32_t)k0, ra);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      reg_fence(ra[i]);
      const int k = k0 + i;
      ra[i] = (k <= dp && (k < ds || k > dw)) ? ra[i] : 0xFF800000u;  // -inf
    }
    tmem_st32u(ts + (uint32_t)k0, ra);
  }
  tmem_wait_st();
}
template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    attn_pp_kernel(const __grid_constant__ CUtensorMap qmap,
                   const __grid_constant__ CUtensorMap kmap,
                   const __grid_constant__ CUtensorMap vmap, const AttnParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  PpSmem& sm = *reinterpret_cast<PpSmem*>(smem_raw +
                                          ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int hidx = blockIdx.y;
  const int h = p.head[hidx];
  const int kvh = h / p.G;
  const int b = blockIdx.z;
  const int rb = gridDim.x - 1 - blockIdx.x;  // heavy (late) row blocks first
  const int m0 = rb * kPRows;
  const int nrows = min(kPRows, p.Lq - m0);
  const int64_t P0 = p.q_pos0 + m0;
  const int64_t Plast = P0 + nrows - 1;
  const Sched sch = make_sched<MODE>(p, P0, Plast);  // the union of both tiles' key tiles

  if (tid == 0) {
    mbar_init(&sm.q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
    }
    for (int q = 0; q < kPQ; ++q) {
      mbar_init(&sm.s_full[q], 1);
      mbar_init(&sm.p_full[q], 4);
      mbar_init(&sm.pv_done[q], 1);
    }
    sm.gave_up = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* gave_up = &sm.gave_up;
  auto t_s = [&](int q) { return tmem + (uint32_t)(q * 256); };
  auto t_o = [&](int q) { return tmem + (uint32_t)(q * 256 + 128); };

  if (warp == kProdWarp) {  // ---------------------------------------- TMA producer
    if (lane == 0) {
      bool ok = true;
      mbar_arrive_expect_tx(&sm.q_full, (uint32_t)(kPQ * kTile));
      for (int q = 0; q < kPQ; ++q) {  // rows past the tensor read as zeros
        tma_load_4d(sm.q[q], &qmap, 0, h, m0 + q * kBM, b * p.bq, &sm.q_full);
        tma_load_4d(sm.q[q] + kHalf, &qmap, 64, h, m0 + q * kBM, b * p.bq, &sm.q_full);
      }
      int n_issued = 0;
      for (int it = 0; it < sch.n; ++it) {
        const int st = it & 1;
        if (!mbar_wait(&sm.kv_empty[st], ((uint32_t)(it >> 1) & 1u) ^ 1u, gave_up)) {
          ok = false;
          break;
        }
        const int j0 = sch.tile(it) * kBN;
        mbar_arrive_expect_tx(&sm.kv_full[st], (uint32_t)(2 * kTile));
        tma_load_4d(sm.k[st], &kmap, 0, kvh, j0, b * p.bk, &sm.kv_full[st]);
        tma_load_4d(sm.k[st] + kHalf, &kmap, 64, kvh, j0, b * p.bk, &sm.kv_full[st]);
        tma_load_4d(sm.v[st], &vmap, 0, kvh, j0, b * p.bk, &sm.kv_full[st]);
        tma_load_4d(sm.v[st] + kHalf, &vmap, 64, kvh, j0, b * p.bk, &sm.kv_full[st]);
        ++n_issued;
      }
      if (!ok) set_status(p.status, RTP_ERR_DEVICE_TIMEOUT, 44);
      for (int k = max(0, n_issued - kStages); k < n_issued; ++k)
        mbar_wait_drain(&sm.kv_full[k & 1], (uint32_t)(k >> 1) & 1u);
      mbar_wait_drain(&sm.q_full, 0u);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {  // ---------------------------------- MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(&sm.q_full, 0u, gave_up);
      int n_pv = 0;
      auto S = [&](int q, int it) {  // S_q = Q_q K(it)^T into the tile's score buffer
        const int st = it & 1;
        if (!mbar_wait(&sm.kv_full[st], (uint32_t)(it >> 1) & 1u, gave_up)) return false;
        // P of the previous key tile is read by its PV MMAs before S overwrites it
        if (it > 0 && !mbar_wait(&sm.pv_done[q], (uint32_t)(it - 1) & 1u, gave_up)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ss(t_s(q), kdesc(sm.q[q], kk), kdesc(sm.k[st], kk), kIdescQK, kk > 0);
        mma_commit(&sm.s_full[q]);
        return true;
      };
      auto PV = [&](int q, int it) {  // O_q += P_q V(it), P read from TMEM
        if (!mbar_wait(&sm.p_full[q], (uint32_t)it & 1u, gave_up)) return false;
        tc_fence_after();
        const int st = it & 1;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ts(t_o(q), t_s(q) + (uint32_t)(kk * 8), vdesc(sm.v[st], kk), kIdescPV,
                      it > 0 || kk > 0);
        mma_commit(&sm.pv_done[q]);
        if (q == kPQ - 1) mma_commit(&sm.kv_empty[st]);  // the stage's last reader
        ++n_pv;
        return true;
      };
      if (ok && sch.n > 0) ok = S(0, 0) && S(1, 0);
      for (int it = 0; ok && it < sch.n; ++it) {
        ok = PV(0, it);
        if (ok && it + 1 < sch.n) ok = S(0, it + 1);
        if (ok) ok = PV(1, it);
        if (ok && it + 1 < sch.n) ok = S(1, it + 1);
      }
      if (!ok) set_status(p.status, RTP_ERR_DEVICE_TIMEOUT, 45);
      if (n_pv > 0)  // the last MMAs are complete before TMEM is released
        for (int q = 0; q < kPQ; ++q)
          mbar_wait_drain(&sm.pv_done[q], (uint32_t)(sch.n - 1) & 1u);
    }
    __syncwarp();
  } else {  // ------------------------------------ softmax: one thread per query row
    const int q = warp >> 2;                  // query tile
    const int r = (warp & 3) * 32 + lane;     // row in the tile = TMEM lane
    const int row = q * kBM + r;              // row in the CTA
    const bool valid = row < nrows;
    const int64_t P = P0 + row;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t ts = t_s(q) + lane_off, to = t_o(q) + lane_off;
    const float c = p.scale_log2;
    float m_used = -INFINITY, l0 = 0.f, l1 = 0.f;  // row sums of keys 0-63 / 64-127 of the tiles
    bool ok = true;
    for (int it = 0; it < sch.n; ++it) {
      const int64_t j0 = (int64_t)sch.tile(it) * kBN;
      ok = ok && mbar_wait_warp(&sm.s_full[q], (uint32_t)it & 1u, gave_up);
      tc_fence_after();
      // key j0 + i is attended to iff i <= dp and (i < ds or i > dw)
      auto clamp_off = [](int64_t d) { return (int)(d < -1 ? -1 : (d > kBN ? kBN : d)); };
      const int dp = clamp_off(P - j0);
      const int ds = MODE == MODE_LOCAL ? clamp_off((int64_t)p.n_sink - j0) : kBN;
      const int dw = MODE == MODE_LOCAL ? clamp_off(P - p.window - j0) : -1;
      // every key of the tile attended to, for every row of the warp: no mask
      const bool wfull = __all_sync(0xffffffffu, dp >= kBN - 1 && (ds >= kBN || dw < 0));
      if (!wfull && ok) pp_mask(ts, dp, ds, dw);
      // the tile's 128 raw scores with one wait; the row max (scale > 0 keeps
      // the order) in the log2 domain
      uint32_t sr[4][32];
      if (ok) {
#pragma unroll
        for (int w = 0; w < 4; ++w) tmem_ld32_nowait(ts + (uint32_t)(w * 32), sr[w]);
        tmem_wait_ld();
      }
      float tm[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) tm[e] = -INFINITY;
#pragma unroll
      for (int w = 0; w < 4; ++w)
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          reg_fence(sr[w][i]);
          reg_fence(sr[w][i + 1]);
          tm[(i >> 1) & 7] =
              max3f(tm[(i >> 1) & 7], __uint_as_float(sr[w][i]), __uint_as_float(sr[w][i + 1]));
        }
      const float smax = fmaxf(fmaxf(fmaxf(tm[0], tm[1]), fmaxf(tm[2], tm[3])),
                               fmaxf(fmaxf(tm[4], tm[5]), fmaxf(tm[6], tm[7])));
      const float tmax = ok ? smax * c : -INFINITY;  // -inf stays -inf
      const float m_new = fmaxf(m_used, tmax);
      const bool first = m_used == -INFINITY && m_new > -INFINITY;  // O and l are still 0
      const bool move = m_used > -INFINITY && m_new > m_used + kRescale;
      float alpha = 1.f;
      if (first) m_used = m_new;
      if (move) {
        alpha = exp2f(m_used - m_new);
        m_used = m_new;
        l0 *= alpha;
        l1 *= alpha;
      }
      // P = 2^(s c - m) rounded to bf16 once, keys 2e, 2e + 1 of the tile into
      // column e (columns already read); the per-half sums gather the fp32
      // values, pair e of a half into slot e % 4 in order of e
      const float msafe = m_used == -INFINITY ? 0.f : m_used;  // masked keys: 2^-inf = 0
      const unsigned long long cc = f2_pack(c, c), mm = f2_pack(-msafe, -msafe);
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {  // keys 64 hf .. 64 hf + 63
        unsigned long long ls[4] = {0ull, 0ull, 0ull, 0ull};  // (+0, +0) pairs
#pragma unroll
        for (int w = 2 * hf; w < 2 * hf + 2; ++w) {  // keys 32 w .. + 31 -> columns 16 w .. + 15
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float x0, x1;
            f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[w][2 * e]), __uint_as_float(sr[w][2 * e + 1])),
                             cc, mm),
                      x0, x1);
            const float p0 = ex2_ftz(x0), p1 = ex2_ftz(x1);
            pk[e] = pack_bf16x2(p0, p1);
            // pair e of the half (16 (w - 2 hf) + e) into slot e % 4: the same slot
            ls[e & 3] = f2_add(ls[e & 3], f2_pack(p0, p1));
          }
          if (ok) tmem_st16u(ts + (uint32_t)(w * 16), pk);
        }
        (hf ? l1 : l0) += fold_sums(ls);
      }
      // O is rescaled (rarely) once the previous key tile's PV MMAs are done (the
      // next PV waits for this tile's P)
      if (it > 0 && __any_sync(0xffffffffu, move)) {
        ok = ok && mbar_wait_warp(&sm.pv_done[q], (uint32_t)(it - 1) & 1u, gave_up);
        tc_fence_after();
        if (ok) {
#pragma unroll 1
          for (int cc = 0; cc < 4; ++cc) {
            float o[32];
            tmem_ld32(to + (uint32_t)(cc * 32), o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tmem_st32(to + (uint32_t)(cc * 32), o);
          }
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.p_full[q]);
    }
    // ---- epilogue: O / l from TMEM, the row's 128 dimensions to global
    if (sch.n > 0)
      ok = ok && mbar_wait_warp(&sm.pv_done[q], (uint32_t)(sch.n - 1) & 1u, gave_up);
    tc_fence_after();
    const float l = l0 + l1;
    const float inv = l > 0.f ? 1.f / l : 0.f;
    uint16_t* orow = p.o + b * p.o_sb + (int64_t)(m0 + row) * p.o_sl + (int64_t)h * kD;
#pragma unroll 1
    for (int cc = 0; cc < 4; ++cc) {
      float o[32];
      if (sch.n > 0) {
        tmem_ld32(to + (uint32_t)(cc * 32), o);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = 0.f;
      }
      if (valid) {
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          uint4 w;
          w.x = pack_bf16x2(o[q4 * 8 + 0] * inv, o[q4 * 8 + 1] * inv);
          w.y = pack_bf16x2(o[q4 * 8 + 2] * inv, o[q4 * 8 + 3] * inv);
          w.z = pack_bf16x2(o[q4 * 8 + 4] * inv, o[q4 * 8 + 5] * inv);
          w.w = pack_bf16x2(o[q4 * 8 + 6] * inv, o[q4 * 8 + 7] * inv);
          *reinterpret_cast<uint4*>(orow + cc * 32 + q4 * 8) = w;
        }
      }
    }
    if (valid && p.lse != nullptr)
      p.lse[((int64_t)b * p.H + h) * p.Lq + m0 + row] =
          l > 0.f ? (m_used + log2f(l)) * kLn2 : -INFINITY;
    if (!ok && row == 0) set_status(p.status, RTP_ERR_DEVICE_TIMEOUT, 46);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// A bf16 [B][L][heads][width] view as a 4-D TMA map {width, heads, L, B} with
// boxes of {box0, 1, 128, 1}; a batch stride of 0 (one tensor shared by every
// batch entry) maps to a single batch coordinate.
bool encode_view(CUtensorMap* map, const rtp_view& v, int width, int heads, int L, int B,
                 int box0, int swizzle, int* batch_mult) {
  const bool shared = v.stride_b == 0 && B > 1;
  *batch_mult = shared ? 0 : 1;
  const uint64_t sl = (uint64_t)v.stride_l * 2;
  const uint64_t sb = !shared && v.stride_b != 0 ? (uint64_t)v.stride_b * 2 : sl * (uint64_t)L;
  const uint64_t dims[4] = {(uint64_t)width, (uint64_t)heads, (uint64_t)L,
                            shared ? 1u : (uint64_t)B};
  const uint64_t strides[3] = {(uint64_t)width * 2, sl, sb};
  const uint32_t box[4] = {(uint32_t)box0, 1, 128, 1};
  return tma_encode_bf16(map, v.ptr, 4, dims, strides, box, swizzle);
}

template <int MODE>
rtp_status launch_tc(AttnParams& prm, int n_heads, const rtp_shape* shape, const rtp_view& q,
                     const rtp_view& k, const rtp_view& v, const rtp_view* q16,
                     const rtp_view* k16, int n_q16, int n_k16, cudaStream_t s) {
  const int B = shape->B;
  if (n_heads == 0 || B == 0 || prm.Lq == 0) return RTP_OK;
  CUtensorMap qm, km, vm, q16m, k16m;
  int bq = 1, bk = 1, bv = 1, b16q = 1, b16k = 1;
  if (!encode_view(&qm, q, kD, shape->H, shape->Lq, B, 64, 128, &bq) ||
      !encode_view(&km, k, kD, shape->Hkv, shape->Lk, B, 64, 128, &bk) ||
      !encode_view(&vm, v, kD, shape->Hkv, shape->Lk, B, 64, 128, &bv))
    return RTP_ERR_CUDA;
  if (MODE == MODE_SPARSE) {
    if (!encode_view(&q16m, *q16, kR, n_q16, shape->Lq, B, kR, 32, &b16q) ||
        !encode_view(&k16m, *k16, kR, n_k16, shape->Lk, B, kR, 32, &b16k))
      return RTP_ERR_CUDA;
    if (b16q != bq || b16k != bk) return RTP_ERR_UNSUPPORTED;  // one batch rule per side
  } else {
    q16m = qm;
    k16m = km;
  }
  if (bk != bv) return RTP_ERR_UNSUPPORTED;
  prm.bq = bq;
  prm.bk = bk;
  static const char* kName[3] = {"attn_prefill_dense", "attn_prefill_local",
                                 "attn_prefill_sparse"};
  if constexpr (MODE != MODE_SPARSE) {  // two query tiles per CTA
    const size_t psmem = sizeof(PpSmem) + 1024;
    if (cudaFuncSetAttribute(attn_pp_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)psmem) != cudaSuccess)
      return RTP_ERR_CUDA;
    dim3 pgrid((prm.Lq + kPRows - 1) / kPRows, n_heads, B);
    if (pgrid.y > 65535 || pgrid.z > 65535) return RTP_ERR_UNSUPPORTED;
    TraceScope tr(kName[MODE], s);
    attn_pp_kernel<MODE><<<pgrid, kThreads, psmem, s>>>(qm, km, vm, prm);
    return check_cuda(cudaGetLastError());
  } else {
  const size_t smem = sizeof(TcSmem) + 1024;
  if (cudaFuncSetAttribute(attn_tc_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return RTP_ERR_CUDA;
  dim3 grid((prm.Lq + kBM - 1) / kBM, n_heads, B);
  if (grid.y > 65535 || grid.z > 65535) return RTP_ERR_UNSUPPORTED;
  TraceScope tr(kName[MODE], s);
  attn_tc_kernel<MODE><<<grid, kThreads, smem, s>>>(qm, km, vm, q16m, k16m, prm);
  return check_cuda(cudaGetLastError());
  }
}

void fill_common(AttnParams& prm, const rtp_shape* shape, const rtp_view& o, float* lse,
                 float softmax_scale, void* ws) {
  memset(&prm, 0, sizeof(prm));
  prm.o = static_cast<uint16_t*>(o.ptr);
  prm.o_sb = o.stride_b;
  prm.o_sl = o.stride_l;
  prm.lse = lse;
  prm.status = static_cast<DevStatus*>(ws);
  prm.Lq = shape->Lq;
  prm.Lk = shape->Lk;
  prm.H = shape->H;
  prm.G = shape->H / shape->Hkv;
  prm.q_pos0 = shape->q_pos0;
  prm.scale_log2 = softmax_scale * kLog2e;
}

}  // namespace

// Entry points used by the C ABI (decode dispatch lives in decode.cu).
rtp_status prefill_local(const rtp_shape* shape, const HeadMap& hm, int window, int n_sink,
                         const rtp_view& q, const rtp_view& k, const rtp_view& v,
                         float scale, const rtp_view& o, float* lse, void* ws, cudaStream_t s) {
  AttnParams prm;
  fill_common(prm, shape, o, lse, scale, ws);
  prm.window = window;
  prm.n_sink = n_sink;
  int n = 0;
  for (int r = 0; r < hm.n_lkv; ++r)
    for (int j = 0; j < hm.G; ++j) prm.head[n++] = (int16_t)(hm.lkv[r] * hm.G + j);
  return launch_tc<MODE_LOCAL>(prm, n, shape, q, k, v, nullptr, nullptr, 0, 0, s);
}

rtp_status prefill_dense(const rtp_shape* shape, const rtp_view& q, const rtp_view& k,
                         const rtp_view& v, float scale, const rtp_view& o, float* lse,
                         void* ws, cudaStream_t s) {
  AttnParams prm;
  fill_common(prm, shape, o, lse, scale, ws);
  for (int h = 0; h < shape->H; ++h) prm.head[h] = (int16_t)h;
  return launch_tc<MODE_DENSE>(prm, shape->H, shape, q, k, v, nullptr, nullptr, 0, 0, s);
}

// Every causal key of the retrieval heads only (p >= 1: the kept set is the
// whole causal prefix), on the dense tile schedule with no indexer recompute.
rtp_status prefill_dense_retrieval(const rtp_shape* shape, const HeadMap& hm, const rtp_view& q,
                                   const rtp_view& k, const rtp_view& v, float scale,
                                   const rtp_view& o, float* lse, void* ws, cudaStream_t s) {
  AttnParams prm;
  fill_common(prm, shape, o, lse, scale, ws);
  for (int hr = 0; hr < hm.n_ret; ++hr) prm.head[hr] = hm.ret_q[hr];
  return launch_tc<MODE_DENSE>(prm, hm.n_ret, shape, q, k, v, nullptr, nullptr, 0, 0, s);
}

rtp_status prefill_sparse(const rtp_shape* shape, const HeadMap& hm, const rtp_view& q,
                          const rtp_view& k, const rtp_view& v, const rtp_view& q16,
                          const rtp_view& k16, const float* thr, const int32_t* jtie,
                          float scale, const rtp_view& o, float* lse, void* ws, cudaStream_t s) {
  AttnParams prm;
  fill_common(prm, shape, o, lse, scale, ws);
  prm.thr = thr;
  prm.jtie = jtie;
  prm.n_ret = hm.n_ret;
  for (int hr = 0; hr < hm.n_ret; ++hr) {
    prm.head[hr] = hm.ret_q[hr];
    prm.slot[hr] = (int16_t)hr;
    prm.k16slot[hr] = hm.ret_k16[hr];
  }
  return launch_tc<MODE_SPARSE>(prm, hm.n_ret, shape, q, k, v, &q16, &k16, hm.n_ret, hm.H_k16,
                                s);
}

}  // namespace rtp
