// attn_prefill.cu -- causal prefill attention tiles for the three head kinds:
//
//   DENSE  every key j <= P (baseline);
//   LOCAL  keys j <= P with j < n_sink or j > P - window ("Local Head Attention
//          Pattern" of the paper-graph-ui summary of arXiv 2605.16928); key
//          tiles outside the sinks and the window are never visited;
//   SPARSE keys j <= P kept by the row's top-p descriptor (thr, jtie) ("Dynamic
//          Top-p Selection Mechanism"): the 16-dim indexer score of every pair is
//          recomputed with the same tensor-core instruction the selection used,
//          so the kept set is reproduced bit for bit.
//
// One CTA = 64 query rows of one head; 4 warps x 16 rows; 64-key tiles of K and
// V double-buffered through shared memory with cp.async; S = QK^T and O += PV on
// the tensor cores (bf16 in, fp32 accumulate), online softmax in registers.
#include "rtp_host.h"

namespace rtp {
namespace {

constexpr int kBM = 64;
constexpr int kBN = 64;
constexpr int kThreads = 128;

enum { MODE_DENSE = 0, MODE_LOCAL = 1, MODE_SPARSE = 2 };

struct AttnParams {
  const uint16_t* q; int64_t q_sb, q_sl;
  const uint16_t* k; int64_t k_sb, k_sl;
  const uint16_t* v; int64_t v_sb, v_sl;
  uint16_t* o; int64_t o_sb, o_sl;
  float* lse;                // [B][H][Lq] or null
  const uint16_t* q16; int64_t q16_sb, q16_sl;
  const uint16_t* k16; int64_t k16_sb, k16_sl;
  const float* thr;          // [B][n_ret][Lq]
  const int32_t* jtie;
  int Lq, Lk, H, G, n_ret;
  int64_t q_pos0;
  int window, n_sink;
  float scale_log2;          // softmax_scale * log2(e)
  int16_t head[kMaxHeads];   // launch head index -> query head
  int16_t slot[kMaxHeads];   // launch head index -> retrieval slot (SPARSE)
  int16_t k16slot[kMaxHeads];// launch head index -> k16 slot (SPARSE)
};

struct AttnSmem {
  uint16_t q[kBM][kD];
  uint16_t k[2][kBN][kD];
  uint16_t v[2][kBN][kD];
  uint16_t k16[2][kBN][kR];
};

// 256-byte rows: 16-byte chunk c of row r lives at chunk c ^ (r & 7).
__device__ __forceinline__ uint32_t swz(const uint16_t (*base)[kD], int r, int chunk) {
  return smem_u32(&base[r][((chunk ^ (r & 7)) << 3)]);
}

__device__ __forceinline__ void load_rows(uint16_t (*dst)[kD], const uint16_t* src_base,
                                          int64_t stride_l, int row0, int nvalid, int tid) {
  // 64 rows x 16 chunks = 1024 chunks / 128 threads
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int c = it * kThreads + tid;
    const int r = c >> 4, ch = c & 15;
    const bool ok = (row0 + r) < nvalid;
    const uint16_t* src = src_base + (int64_t)(ok ? row0 + r : 0) * stride_l + ch * 8;
    cp_async16(swz(dst, r, ch), src, ok);
  }
}

template <int MODE>
__global__ void __launch_bounds__(kThreads) attn_prefill_kernel(const AttnParams p) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  AttnSmem& sm = *reinterpret_cast<AttnSmem*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int hidx = blockIdx.y;
  const int h = p.head[hidx];
  const int kvh = h / p.G;
  const int b = blockIdx.z;
  const int tile = gridDim.x - 1 - blockIdx.x;
  const int m0 = tile * kBM;
  const int nrows = min(kBM, p.Lq - m0);
  const int64_t P0 = p.q_pos0 + m0;               // position of CTA row 0
  const int64_t Plast = P0 + nrows - 1;

  const uint16_t* qb = p.q + b * p.q_sb + (int64_t)h * kD;
  const uint16_t* kb = p.k + b * p.k_sb + (int64_t)kvh * kD;
  const uint16_t* vb = p.v + b * p.v_sb + (int64_t)kvh * kD;

  // ---- key-tile schedule
  int t_begin = 0, t_sink_end = 0, t_win_begin = 0;
  const int t_end = (int)(Plast / kBN);             // inclusive
  if (MODE == MODE_LOCAL) {
    t_sink_end = (p.n_sink + kBN - 1) / kBN;         // tiles [0, t_sink_end)
    const int64_t wlo = P0 - p.window + 1;           // lowest window key of row 0
    t_win_begin = (int)((wlo > 0 ? wlo : 0) / kBN);
    if (t_win_begin < t_sink_end) t_win_begin = t_sink_end;
  }
  auto nth_tile = [&](int it) -> int {
    if (MODE != MODE_LOCAL) return t_begin + it;
    return it < t_sink_end ? it : t_win_begin + (it - t_sink_end);
  };
  int n_iter;
  if (MODE == MODE_LOCAL) {
    const int sinks = min(t_sink_end, t_end + 1);
    n_iter = sinks + max(0, t_end - t_win_begin + 1);
    t_sink_end = sinks;
  } else {
    n_iter = t_end + 1;
  }

  // ---- Q tile -> registers
  load_rows(sm.q, qb + (int64_t)m0 * p.q_sl, p.q_sl, 0, nrows, tid);
  cp_async_commit();

  const uint16_t* k16b = nullptr;
  uint32_t qa16[4] = {0, 0, 0, 0};
  float tA = 0.f, tB = 0.f;
  int jA = 0, jB = 0;
  const int rA = warp * 16 + g, rB = rA + 8;
  if (MODE == MODE_SPARSE) {
    const int slot = p.slot[hidx];
    k16b = p.k16 + b * p.k16_sb + (int64_t)p.k16slot[hidx] * kR;
    const uint16_t* q16b = p.q16 + b * p.q16_sb + (int64_t)slot * kR;
    auto ld = [&](int r, int d) -> uint32_t {
      if (r >= nrows) return 0u;
      return *reinterpret_cast<const uint32_t*>(q16b + (int64_t)(m0 + r) * p.q16_sl + d);
    };
    qa16[0] = ld(rA, 2 * t);
    qa16[1] = ld(rB, 2 * t);
    qa16[2] = ld(rA, 2 * t + 8);
    qa16[3] = ld(rB, 2 * t + 8);
    const int64_t ob = ((int64_t)b * p.n_ret + slot) * p.Lq + m0;
    if (rA < nrows) { tA = p.thr[ob + rA]; jA = p.jtie[ob + rA]; }
    if (rB < nrows) { tB = p.thr[ob + rB]; jB = p.jtie[ob + rB]; }
  }

  auto load_kv = [&](int it, int buf) {
    const int kt = nth_tile(it);
    load_rows(sm.k[buf], kb + (int64_t)kt * kBN * p.k_sl, p.k_sl, 0, p.Lk - kt * kBN, tid);
    load_rows(sm.v[buf], vb + (int64_t)kt * kBN * p.v_sl, p.v_sl, 0, p.Lk - kt * kBN, tid);
    if (MODE == MODE_SPARSE) {
      const int key = tid >> 1, ch = tid & 1;
      const int j = kt * kBN + key;
      const bool ok = j < p.Lk;
      cp_async16(smem_u32(&sm.k16[buf][key][(ch ^ ((key >> 2) & 1)) * 8]),
                 k16b + (int64_t)(ok ? j : 0) * p.k16_sl + ch * 8, ok);
    }
  };

  if (n_iter > 0) load_kv(0, 0);
  cp_async_commit();
  cp_async_wait<1>();
  __syncthreads();
  uint32_t qa[8][4];
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const int r = warp * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
    ldmatrix_x4(qa[kk], swz(sm.q, r, 2 * kk + (lane >> 4)));
  }

  float oacc[16][4];
#pragma unroll
  for (int d = 0; d < 16; ++d)
#pragma unroll
    for (int e = 0; e < 4; ++e) oacc[d][e] = 0.f;
  float mrow[2] = {-INFINITY, -INFINITY};
  float lrow[2] = {0.f, 0.f};
  const int64_t PA = P0 + rA, PB = P0 + rB;
  const int64_t warp_P0 = P0 + warp * 16;
  const int64_t warp_Plast = P0 + min(warp * 16 + 15, nrows - 1);
  const bool warp_has_rows = warp * 16 < nrows;

  for (int it = 0; it < n_iter; ++it) {
    const int buf = it & 1;
    if (it + 1 < n_iter) {
      load_kv(it + 1, buf ^ 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const int kt = nth_tile(it);
    const int64_t j0 = (int64_t)kt * kBN;
    bool run = warp_has_rows && j0 <= warp_Plast;
    if (MODE == MODE_LOCAL) {
      // skip tiles entirely outside this warp's sinks+window
      const bool in_sink = j0 < p.n_sink;
      const bool in_win = j0 + kBN - 1 > warp_P0 - p.window;
      run = run && (in_sink || in_win);
    }
    // sparse: indexer-score predicate first; skip the tile if nothing is kept
    uint32_t keep[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (MODE == MODE_SPARSE && run) {
      bool any = false;
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        const int q = lane >> 3;
        const int key = np * 16 + (lane & 7) + 8 * (q >> 1);
        const int ch = q & 1;
        uint32_t r[4];
        ldmatrix_x4(r, smem_u32(&sm.k16[buf][key][(ch ^ ((key >> 2) & 1)) * 8]));
        float s0[4], s1[4];
        mma16816_zero(s0, qa16, r[0], r[1]);
        mma16816_zero(s1, qa16, r[2], r[3]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const bool hi = e >= 2;
          const float th = hi ? tB : tA;
          const int jt = hi ? jB : jA;
          const int64_t P = hi ? PB : PA;
          const int64_t ja = j0 + (2 * np) * 8 + 2 * t + (e & 1);
          const int64_t jb = ja + 8;
          const float sa = s0[e] + 0.0f, sb = s1[e] + 0.0f;
          const bool ka = ja <= P && (sa > th || (sa == th && ja <= jt));
          const bool kb2 = jb <= P && (sb > th || (sb == th && jb <= jt));
          keep[2 * np] |= (uint32_t)ka << e;
          keep[2 * np + 1] |= (uint32_t)kb2 << e;
          any = any || ka || kb2;
        }
      }
      run = __any_sync(0xffffffffu, any);
    }
    if (run) {
      float s[8][4];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) s[nt][e] = 0.f;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
        for (int np = 0; np < 4; ++np) {
          const int q = lane >> 3;
          const int key = np * 16 + (lane & 7) + 8 * (q >> 1);
          uint32_t r[4];
          ldmatrix_x4(r, swz(sm.k[buf], key, 2 * kk + (q & 1)));
          mma16816(s[2 * np], qa[kk], r[0], r[1], s[2 * np]);
          mma16816(s[2 * np + 1], qa[kk], r[2], r[3], s[2 * np + 1]);
        }
      }
      // mask + scale into the log2 domain
      const bool full_tile = (MODE == MODE_DENSE && j0 + kBN - 1 <= warp_P0) ||
                             (MODE == MODE_LOCAL && j0 + kBN - 1 <= warp_P0 &&
                              j0 > warp_Plast - p.window);
      float tmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const bool hi = e >= 2;
          bool ok = true;
          if (!full_tile) {
            const int64_t j = j0 + nt * 8 + 2 * t + (e & 1);
            const int64_t P = hi ? PB : PA;
            if (MODE == MODE_DENSE) ok = j <= P;
            else if (MODE == MODE_LOCAL) ok = j <= P && (j < p.n_sink || j > P - p.window);
            else ok = (keep[nt] >> e) & 1u;
          }
          const float x = ok ? s[nt][e] * p.scale_log2 : -INFINITY;
          s[nt][e] = x;
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
      // probabilities rounded to bf16 once: the same values feed PV and the
      // normaliser, so the output stays an exact convex combination of them
      uint32_t pp[8][2];
      float ls[2] = {0.f, 0.f};
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        float pr[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          pr[e] = (s[nt][e] == -INFINITY) ? 0.f : exp2f(s[nt][e] - mrow[e >= 2]);
        pp[nt][0] = pack_bf16x2(pr[0], pr[1]);
        pp[nt][1] = pack_bf16x2(pr[2], pr[3]);
        ls[0] += bf16_lo(pp[nt][0]) + bf16_hi(pp[nt][0]);
        ls[1] += bf16_lo(pp[nt][1]) + bf16_hi(pp[nt][1]);
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
      // O += P V
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint32_t pa[4] = {pp[2 * kk][0], pp[2 * kk][1], pp[2 * kk + 1][0],
                                pp[2 * kk + 1][1]};
#pragma unroll
        for (int dp = 0; dp < 8; ++dp) {
          const int q = lane >> 3;
          const int key = kk * 16 + (lane & 7) + 8 * (q & 1);
          uint32_t r[4];
          ldmatrix_x4_trans(r, swz(sm.v[buf], key, 2 * dp + (q >> 1)));
          mma16816(oacc[2 * dp], pa, r[0], r[1], oacc[2 * dp]);
          mma16816(oacc[2 * dp + 1], pa, r[2], r[3], oacc[2 * dp + 1]);
        }
      }
    }
    __syncthreads();
  }

  // ---- epilogue: normalise, stage through shared memory, 16-byte stores
  float inv[2];
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    const float l = quad_sum(lrow[hh]);
    inv[hh] = l > 0.f ? 1.f / l : 0.f;
    if (p.lse != nullptr && t == 0) {
      const int r = hh ? rB : rA;
      if (r < nrows) {
        const float lse = l > 0.f ? (mrow[hh] + log2f(l)) * kLn2 : -INFINITY;
        p.lse[((int64_t)b * p.H + h) * p.Lq + m0 + r] = lse;
      }
    }
  }
#pragma unroll
  for (int d = 0; d < 16; ++d) {
    const int col = d * 8 + 2 * t;
    const uint32_t lo = pack_bf16x2(oacc[d][0] * inv[0], oacc[d][1] * inv[0]);
    const uint32_t hi = pack_bf16x2(oacc[d][2] * inv[1], oacc[d][3] * inv[1]);
    *reinterpret_cast<uint32_t*>(&sm.q[rA][(((col >> 3) ^ (rA & 7)) << 3) + (col & 7)]) = lo;
    *reinterpret_cast<uint32_t*>(&sm.q[rB][(((col >> 3) ^ (rB & 7)) << 3) + (col & 7)]) = hi;
  }
  __syncthreads();
  uint16_t* ob = p.o + b * p.o_sb + (int64_t)h * kD;
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int c = it * kThreads + tid;
    const int r = c >> 4, ch = c & 15;
    if (r < nrows) {
      const uint4 val = *reinterpret_cast<const uint4*>(&sm.q[r][((ch ^ (r & 7)) << 3)]);
      *reinterpret_cast<uint4*>(ob + (int64_t)(m0 + r) * p.o_sl + ch * 8) = val;
    }
  }
}

template <int MODE>
rtp_status launch(const AttnParams& prm, int n_heads, int B, cudaStream_t s) {
  if (n_heads == 0 || B == 0 || prm.Lq == 0) return RTP_OK;
  const size_t smem = sizeof(AttnSmem);
  if (cudaFuncSetAttribute(attn_prefill_kernel<MODE>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return RTP_ERR_CUDA;
  dim3 grid((prm.Lq + kBM - 1) / kBM, n_heads, B);
  if (grid.y > 65535 || grid.z > 65535) return RTP_ERR_UNSUPPORTED;
  static const char* kName[3] = {"attn_prefill_dense", "attn_prefill_local", "attn_prefill_sparse"};
  TraceScope tr(kName[MODE], s);
  attn_prefill_kernel<MODE><<<grid, kThreads, smem, s>>>(prm);
  return check_cuda(cudaGetLastError());
}

void fill_common(AttnParams& prm, const rtp_shape* shape, const rtp_view& q, const rtp_view& k,
                 const rtp_view& v, const rtp_view& o, float* lse, float softmax_scale) {
  memset(&prm, 0, sizeof(prm));
  prm.q = static_cast<const uint16_t*>(q.ptr); prm.q_sb = q.stride_b; prm.q_sl = q.stride_l;
  prm.k = static_cast<const uint16_t*>(k.ptr); prm.k_sb = k.stride_b; prm.k_sl = k.stride_l;
  prm.v = static_cast<const uint16_t*>(v.ptr); prm.v_sb = v.stride_b; prm.v_sl = v.stride_l;
  prm.o = static_cast<uint16_t*>(o.ptr); prm.o_sb = o.stride_b; prm.o_sl = o.stride_l;
  prm.lse = lse;
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
                         float scale, const rtp_view& o, float* lse, cudaStream_t s) {
  AttnParams prm;
  fill_common(prm, shape, q, k, v, o, lse, scale);
  prm.window = window;
  prm.n_sink = n_sink;
  int n = 0;
  for (int r = 0; r < hm.n_lkv; ++r)
    for (int j = 0; j < hm.G; ++j) prm.head[n++] = (int16_t)(hm.lkv[r] * hm.G + j);
  return launch<MODE_LOCAL>(prm, n, shape->B, s);
}

rtp_status prefill_dense(const rtp_shape* shape, const rtp_view& q, const rtp_view& k,
                         const rtp_view& v, float scale, const rtp_view& o, float* lse,
                         cudaStream_t s) {
  AttnParams prm;
  fill_common(prm, shape, q, k, v, o, lse, scale);
  for (int h = 0; h < shape->H; ++h) prm.head[h] = (int16_t)h;
  return launch<MODE_DENSE>(prm, shape->H, shape->B, s);
}

rtp_status prefill_sparse(const rtp_shape* shape, const HeadMap& hm, const rtp_view& q,
                          const rtp_view& k, const rtp_view& v, const rtp_view& q16,
                          const rtp_view& k16, const float* thr, const int32_t* jtie,
                          float scale, const rtp_view& o, float* lse, cudaStream_t s) {
  AttnParams prm;
  fill_common(prm, shape, q, k, v, o, lse, scale);
  prm.q16 = static_cast<const uint16_t*>(q16.ptr);
  prm.q16_sb = q16.stride_b;
  prm.q16_sl = q16.stride_l;
  prm.k16 = static_cast<const uint16_t*>(k16.ptr);
  prm.k16_sb = k16.stride_b;
  prm.k16_sl = k16.stride_l;
  prm.thr = thr;
  prm.jtie = jtie;
  prm.n_ret = hm.n_ret;
  for (int hr = 0; hr < hm.n_ret; ++hr) {
    prm.head[hr] = hm.ret_q[hr];
    prm.slot[hr] = (int16_t)hr;
    prm.k16slot[hr] = hm.ret_k16[hr];
  }
  return launch<MODE_SPARSE>(prm, hm.n_ret, shape->B, s);
}

}  // namespace rtp
