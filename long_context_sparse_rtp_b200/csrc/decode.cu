// decode.cu -- single-token decode: retrieval heads (rtp_sparse_attn_decode) and
// the range-mode decode attention used by local and dense heads.
//
// Retrieval decode for one query token per batch entry ("Dynamic Top-p
// Selection Mechanism" and the decode flow of the paper-graph-ui summary of
// arXiv 2605.16928), per kv group of G query heads: the scores, the exact cut
// and the kept-key union list come from decode_select.cu; this file holds the
// attention over that list and over sink + window ranges:
//   attend   split-KV over the list (or the range): gathered K/V rows staged in
//            shared memory with 16-byte cp.async, tensor-core QK^T / PV with the
//            G heads as mma rows, per-head masks, online softmax, one partial
//            (m, l, o) per split;
//   merge    a second kernel, one CTA per (batch, kv group, head), combines the
//            splits in split order.
#include <algorithm>

#include "rtp_host.h"

namespace rtp {

rtp_status prefill_local(const rtp_shape*, const HeadMap&, int, int, const rtp_view&,
                         const rtp_view&, const rtp_view&, float, const rtp_view&, float*, void*,
                         cudaStream_t);
rtp_status prefill_dense(const rtp_shape*, const rtp_view&, const rtp_view&, const rtp_view&,
                         float, const rtp_view&, float*, void*, cudaStream_t);
rtp_status prefill_dense_retrieval(const rtp_shape*, const HeadMap&, const rtp_view&,
                                   const rtp_view&, const rtp_view&, float, const rtp_view&,
                                   float*, void*, cudaStream_t);
rtp_status prefill_sparse(const rtp_shape*, const HeadMap&, const rtp_view&, const rtp_view&,
                          const rtp_view&, const rtp_view&, const rtp_view&, const float*,
                          const int32_t*, float, const rtp_view&, float*, void*, cudaStream_t);

namespace {

// ------------------------------------------------------------------ 4. attend
struct DecAttnParams {
  const uint16_t* q; int64_t q_sb;       // query row of each batch entry
  const uint16_t* k; int64_t k_sb, k_sl;
  const uint16_t* v; int64_t v_sb, v_sl;
  uint16_t* o; int64_t o_sb;
  float* lse; int64_t lse_sb;            // lse[b*lse_sb + h] (Lq == 1)
  float scale_log2;
  int G, groups, n_splits;
  // list mode: per kv group, per chunk of kDecChunk tokens, an ordered list of
  // {token, kept-head bits | candidate-head bits << 16}; candidate bits are
  // settled here with the exact predicate on the stored indexer score.
  const uint2* list; const int32_t* lcount; int Lk_pad, n_chunks;
  const float* scores;                    // [rows][Lk_pad]
  const RowRes* rowres;                   // [rows]: t, jtie of each retrieval row
  int n_ret;
  // range mode
  int64_t P; int n_sink_eff; int64_t win_lo; int64_t n_keys; int keys_per_split;
  float* part;                            // [B*groups][n_splits][16][2+128]
  int16_t kvh[kMaxHeads];                 // group -> kv head (its query heads in q, o, lse)
  int16_t kslot[kMaxHeads];               // group -> head slot of the k / v views
  // ring cache (range mode): position j >= ring_sink lives in row
  // ring_sink + (j - ring_sink) % ring_w of k / v; ring_w == 0: row j
  int ring_w, ring_sink;
};

constexpr int kDecThreads = 128;
constexpr int kTile = 64;
constexpr int kMaxSplits = kDecMaxSplits;  // the merge keeps 3 x 256 x 16 floats in K/V smem
constexpr int kRound = 512;  // list entries a CTA resolves into shared memory at once

struct DecSmem {
  uint16_t q[16][kD];
  uint16_t k[2][kTile][kD];
  uint16_t v[2][kTile][kD];
  uint32_t mask[2][kTile];
  float wm[4][16], wl[4][16];
  float t[16];
  int jt[16];
  int etok[kRound];        // list mode: resolved tokens and head masks of this round
  uint32_t emask[kRound];
  float lsum[16], mmax[16];
  int wsc[kDecThreads / 32];
  int loffs[1];  // list mode: n_chunks + 1 entries (dynamic tail)
};

__device__ __forceinline__ uint32_t dswz(const uint16_t (*base)[kD], int r, int chunk) {
  return smem_u32(&base[r][((chunk ^ (r & 7)) << 3)]);
}

template <bool LIST>
__global__ void __launch_bounds__(kDecThreads) dec_attn_kernel(const DecAttnParams p) {
  griddep_wait();  // launched as a dependent of the previous kernel
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
  int n_entries = 0;
  if (LIST) {  // an equal share of the group's list entries
    // exclusive prefix of the chunk counts (block scan)
    const int nc = p.n_chunks;
    const int32_t* lc = p.lcount + (int64_t)gg * nc;
    const int per = (nc + kDecThreads - 1) / kDecThreads;  // <= 16 (nc <= 2048)
    const int c0 = tid * per, c1 = min(nc, c0 + per);
    int cv[16];
    int seg = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      cv[i] = (c0 + i < c1) ? lc[c0 + i] : 0;
      seg += cv[i];
    }
    int inc = seg;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    if (lane == 31) sm.wsc[warp] = inc;
    __syncthreads();
    int run = inc - seg;
    for (int w2 = 0; w2 < warp; ++w2) run += sm.wsc[w2];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if (c0 + i < c1) sm.loffs[c0 + i] = run;
      run += cv[i];
    }
    __syncthreads();
    if (tid == kDecThreads - 1) {
      int tot = 0;
      for (int w2 = 0; w2 < kDecThreads / 32; ++w2) tot += sm.wsc[w2];
      sm.loffs[nc] = tot;
    }
    __syncthreads();
    const int64_t total = sm.loffs[p.n_chunks];
    e_begin = total * split / p.n_splits;
    e_end = total * (split + 1) / p.n_splits;
    n_entries = (int)(e_end - e_begin);
  } else {
    e_begin = (int64_t)split * p.keys_per_split;
    e_end = min(p.n_keys, e_begin + p.keys_per_split);
    n_entries = (int)max((int64_t)0, e_end - e_begin);
  }
  const uint16_t* kb = p.k + b * p.k_sb + (int64_t)p.kslot[grp] * kD;
  const uint16_t* vb = p.v + b * p.v_sb + (int64_t)p.kslot[grp] * kD;

  if (LIST) {
    if (tid < G) {
      const RowRes rr = p.rowres[b * p.n_ret + grp * G + tid];
      sm.t[tid] = rr.t;
      sm.jt[tid] = rr.jtie;
    }
    __syncthreads();
  }
  // list mode: entries are resolved a round at a time, all loads in flight together
  auto resolve_round = [&](int r0, int nr) {
#pragma unroll 4
    for (int e = tid; e < nr; e += kDecThreads) {
      const int ge = (int)(e_begin + r0 + e);
      int lo = 0, hi = p.n_chunks - 1;  // last chunk c with loffs[c] <= ge
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (sm.loffs[mid] <= ge) lo = mid; else hi = mid - 1;
      }
      const uint2 x = p.list[(int64_t)gg * p.Lk_pad + lo * kDecChunk + (ge - sm.loffs[lo])];
      uint32_t keep = x.y & 0xFFFFu;
      uint32_t cand = x.y >> 16;
      while (cand) {  // exact predicate: s > t, or s == t and j <= jtie
        const int hh = __ffs(cand) - 1;
        cand &= cand - 1;
        const float sc = p.scores[(int64_t)(b * p.n_ret + grp * G + hh) * p.Lk_pad + x.x];
        if (sc > sm.t[hh] || (sc == sm.t[hh] && (int)x.x <= sm.jt[hh])) keep |= 1u << hh;
      }
      sm.etok[e] = (int)x.x;
      sm.emask[e] = keep;
    }
  };
  // range mode: entry e -> key
  auto range_key = [&](int e) -> int64_t {
    const int64_t ve = e_begin + e;
    return ve < p.n_sink_eff ? ve : p.win_lo + (ve - p.n_sink_eff);
  };
  int round0 = 0, n_round = n_entries;  // entries [round0, round0 + n_round) of this pass
  auto load_tile = [&](int it, int buf) {
    // 64 rows x 16 chunks for K and for V: 16 cp.async per thread
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int c = u * kDecThreads + tid;
      const int r = c >> 4, ch = c & 15;
      const int e = it * kTile + r;  // within the round
      const bool ok = e < n_round;
      int64_t j = 0;
      uint32_t msk = 0;
      if (ok) {
        if (LIST) {
          j = sm.etok[e];
          msk = sm.emask[e];
        } else {
          j = range_key(round0 + e);
          if (p.ring_w > 0 && j >= p.ring_sink)
            j = p.ring_sink + (int64_t)((uint32_t)(j - p.ring_sink) % (uint32_t)p.ring_w);
          msk = allmask;
        }
      }
      cp_async16(dswz(sm.k[buf], r, ch), kb + j * p.k_sl + ch * 8, ok);
      cp_async16(dswz(sm.v[buf], r, ch), vb + j * p.v_sl + ch * 8, ok);
      if (ch == 0) sm.mask[buf][r] = ok ? msk : 0u;
    }
  };

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

  for (round0 = 0; round0 < max(n_entries, 1); round0 += (LIST ? kRound : max(n_entries, 1))) {
  n_round = LIST ? min(kRound, n_entries - round0) : n_entries;
  if (LIST) {
    __syncthreads();  // the previous round's entries are no longer read
    resolve_round(round0, n_round);
    __syncthreads();
  }
  const int n_tiles = (n_round + kTile - 1) / kTile;
  if (n_tiles > 0) load_tile(0, 0);
  cp_async_commit();
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

  }  // rounds

  // ---- merge the 4 warps (each saw a quarter of every tile); the K/V staging
  // buffers are free now and hold the warps' partial outputs
  float (*wo)[16][kD] = reinterpret_cast<float (*)[16][kD]>(&sm.k[0][0][0]);
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
    wo[warp][g][col] = oacc[d][0];
    wo[warp][g][col + 1] = oacc[d][1];
    wo[warp][g + 8][col] = oacc[d][2];
    wo[warp][g + 8][col + 1] = oacc[d][3];
  }
  __syncthreads();
  float* part = p.part + ((int64_t)gg * p.n_splits + split) * 16 * kPartRow;
  for (int x = tid; x < 16 * kD; x += kDecThreads) {
    const int r = x / kD, d = x % kD;
    float M = -INFINITY;
    for (int w = 0; w < 4; ++w) M = fmaxf(M, sm.wm[w][r]);
    float o = 0.f, l = 0.f;
    if (M != -INFINITY) {
      for (int w = 0; w < 4; ++w) {
        const float f = (sm.wm[w][r] == -INFINITY) ? 0.f : exp2f(sm.wm[w][r] - M);
        o += f * wo[w][r][d];
        l += f * sm.wl[w][r];
      }
    }
    part[r * kPartRow + 4 + d] = o;
    if (d == 0) {
      part[r * kPartRow] = M;
      part[r * kPartRow + 1] = l;
    }
  }
}

// Merge of one (batch, kv group, head)'s split partials by one warp: lane i
// owns dimensions 4i .. 4i + 3 and sums the splits in split order; the mass l is
// a per-lane sum in split order followed by a fixed butterfly, so the result
// does not depend on which split finished last.  Launched after the split
// kernel on the same stream.
__global__ void __launch_bounds__(32) dec_split_merge_kernel(const DecAttnParams p) {
  griddep_wait();  // launched as a dependent of the previous kernel
  __shared__ float fs[kMaxSplits];
  const int gg = blockIdx.x, r = blockIdx.y;  // b * groups + group, head of the group
  const int b = gg / p.groups, grp = gg % p.groups;
  const int lane = threadIdx.x;
  const int64_t sstride = 16 * kPartRow;  // floats between consecutive splits
  const float* pg = p.part + (int64_t)gg * p.n_splits * sstride + (int64_t)r * kPartRow;
  const int ns = min(p.n_splits, kMaxSplits);
  float M = -INFINITY;
  for (int sp = lane; sp < ns; sp += 32) M = fmaxf(M, __ldcg(pg + sp * sstride));
  M = warp_max(M);
  float l = 0.f;
  for (int sp = lane; sp < ns; sp += 32) {
    const float ms = __ldcg(pg + sp * sstride), ls = __ldcg(pg + sp * sstride + 1);
    const float f = (ms == -INFINITY) ? 0.f : exp2f(ms - M);
    fs[sp] = f;
    l += f * ls;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
  __syncwarp();
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  const float* po = pg + 4 + 4 * lane;
  int sp = 0;
  for (; sp + 8 <= ns; sp += 8) {  // eight independent 16-byte loads in flight
    float4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = __ldcg(reinterpret_cast<const float4*>(po + (sp + u) * sstride));
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float f = fs[sp + u];
      acc.x += f * v[u].x;
      acc.y += f * v[u].y;
      acc.z += f * v[u].z;
      acc.w += f * v[u].w;
    }
  }
  for (; sp < ns; ++sp) {
    const float4 v = __ldcg(reinterpret_cast<const float4*>(po + sp * sstride));
    const float f = fs[sp];
    acc.x += f * v.x;
    acc.y += f * v.y;
    acc.z += f * v.z;
    acc.w += f * v.w;
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
  const int h = p.kvh[grp] * p.G + r;
  uint2 w;
  w.x = pack_bf16x2(acc.x * inv, acc.y * inv);
  w.y = pack_bf16x2(acc.z * inv, acc.w * inv);
  *reinterpret_cast<uint2*>(p.o + b * p.o_sb + (int64_t)h * kD + 4 * lane) = w;
  if (lane == 0 && p.lse != nullptr)
    p.lse[b * p.lse_sb + h] = l > 0.f ? (M + log2f(l)) * kLn2 : -INFINITY;
}

template <bool LIST>
rtp_status launch_dec_attn(const DecAttnParams& prm, int B, cudaStream_t s) {
  const size_t smem = sizeof(DecSmem) + (LIST ? (size_t)(prm.n_chunks + 1) * 4 : 0);
  if (cudaFuncSetAttribute(dec_attn_kernel<LIST>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return RTP_ERR_CUDA;
  dim3 grid(prm.n_splits, B * prm.groups);
  if (grid.y > 65535) return RTP_ERR_UNSUPPORTED;
  rtp_status st;
  {
    TraceScope tr(LIST ? "dec_attn_list" : "dec_attn_range", s);
    if ((st = check_cuda(launch_dependent(dec_attn_kernel<LIST>, grid, dim3(kDecThreads), smem, s,
                                          prm))) != RTP_OK)
      return st;
  }
  TraceScope tr(LIST ? "dec_merge_list" : "dec_merge_range", s);
  return check_cuda(launch_dependent(dec_split_merge_kernel, dim3(B * prm.groups, prm.G), dim3(32),
                                     0, s, prm));
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
// With ring_w > 0 the k / v views are ring caches holding only these groups'
// heads (slot i = group i) of n_sink + ring_w rows.
rtp_status decode_range(const rtp_shape* shape, const int16_t* kv_heads, int n_groups,
                        int window, int n_sink, const rtp_view& q, const rtp_view& k,
                        const rtp_view& v, float scale, const rtp_view& o, float* lse,
                        void* ws, size_t ws_bytes, cudaStream_t s, int ring_w = 0) {
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
  prm.keys_per_split = L.keys_per_split;
  prm.part = reinterpret_cast<float*>(static_cast<char*>(ws) + L.part);
  prm.ring_w = ring_w;
  prm.ring_sink = n_sink;
  for (int i = 0; i < n_groups; ++i) {
    prm.kvh[i] = kv_heads[i];
    prm.kslot[i] = ring_w > 0 ? (int16_t)i : kv_heads[i];
  }
  return launch_dec_attn<false>(prm, shape->B, s);
}

// ------------------------------------------------------------------ ring cache writes
// Copies the local kv heads of source positions into a ring cache: position
// j < n_sink to row j, position j >= n_sink to row n_sink + (j - n_sink) % window.
// Only the positions a later query can still see are copied: the sinks and the
// last `window` positions of the range (an earlier one would be overwritten).
struct RingWriteParams {
  const uint16_t* k; int64_t k_sb, k_sl;  // source row i holds position pos0 + i
  const uint16_t* v; int64_t v_sb, v_sl;
  uint16_t* kr; int64_t kr_sb, kr_sl;     // ring [B][n_sink + window][n_lkv][128]
  uint16_t* vr; int64_t vr_sb, vr_sl;
  int64_t pos0, a0, a1, w0, w1;           // sink positions [a0, a1), window [w0, w1)
  int n_sink, window, n_lkv;
  int16_t lkv[kMaxHeads];
};

constexpr int kRingThreads = 256;

__global__ void __launch_bounds__(kRingThreads) ring_write_kernel(const RingWriteParams p) {
  const int64_t e = (int64_t)blockIdx.x * kRingThreads + threadIdx.x;
  const int b = blockIdx.y;
  const int chunk = (int)(e & 15);               // 16 bytes of a 256-byte head row
  const int64_t rest = e >> 4;
  const int i = (int)(rest % p.n_lkv);
  const int64_t m = rest / p.n_lkv;
  const int64_t n1 = p.a1 - p.a0;
  const int64_t j = m < n1 ? p.a0 + m : p.w0 + (m - n1);
  if (m >= n1 && j >= p.w1) return;
  const int64_t slot =
      j < p.n_sink ? j : p.n_sink + (int64_t)((uint64_t)(j - p.n_sink) % (uint64_t)p.window);
  const int64_t src_k = b * p.k_sb + (j - p.pos0) * p.k_sl + (int64_t)p.lkv[i] * kD + chunk * 8;
  const int64_t src_v = b * p.v_sb + (j - p.pos0) * p.v_sl + (int64_t)p.lkv[i] * kD + chunk * 8;
  const int64_t dk = b * p.kr_sb + slot * p.kr_sl + (int64_t)i * kD + chunk * 8;
  const int64_t dv = b * p.vr_sb + slot * p.vr_sl + (int64_t)i * kD + chunk * 8;
  *reinterpret_cast<uint4*>(p.kr + dk) = *reinterpret_cast<const uint4*>(p.k + src_k);
  *reinterpret_cast<uint4*>(p.vr + dv) = *reinterpret_cast<const uint4*>(p.v + src_v);
}

}  // namespace

rtp_status decode_list_attention(const rtp_shape* shape, const HeadMap& hm, const rtp_view& q,
                                 const rtp_view& k, const rtp_view& v, float scale,
                                 const rtp_view& o, float* lse, const DecodeLists& lists,
                                 cudaStream_t s) {
  DecAttnParams prm;
  fill_dec_common(prm, shape, q, k, v, o, lse, scale);
  prm.groups = hm.n_rkv;
  prm.list = lists.list;
  prm.lcount = lists.lcount;
  prm.Lk_pad = lists.Lk_pad;
  prm.n_chunks = lists.n_chunks;
  prm.n_splits = lists.n_splits;
  prm.scores = lists.scores;
  prm.rowres = lists.rowres;
  prm.n_ret = hm.n_ret;
  prm.part = lists.part;
  for (int i = 0; i < hm.n_rkv; ++i) prm.kvh[i] = prm.kslot[i] = hm.rkv[i];
  return launch_dec_attn<true>(prm, shape->B, s);
}

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
    case RTP_OP_TOPP_SELECT: {
      const size_t t = select_ws_layout().total;
      return t > 0 ? t : kStatusBytes;
    }
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
  return prefill_local(shape, hm, window, n_sink, q, k, v, softmax_scale, o, lse, ws, s);
}

extern "C" rtp_status rtp_local_ring_write(const rtp_shape* shape, const uint8_t* kv_role,
                                           int32_t window, int32_t n_sink, rtp_view k,
                                           rtp_view v, rtp_view k_ring, rtp_view v_ring,
                                           rtp_stream_t stream) {
  rtp_status st = check_shape(shape);
  if (st != RTP_OK) return st;
  HeadMap hm;
  if ((st = make_headmap(shape, kv_role, 0, &hm)) != RTP_OK) return st;
  if (window < 1 || n_sink < 0) return RTP_ERR_INVALID_ARG;
  if (shape->B == 0 || shape->Lq == 0 || hm.n_lkv == 0) return RTP_OK;
  if ((st = check_view(k, shape->Hkv, kD, true)) != RTP_OK) return st;
  if ((st = check_view(v, shape->Hkv, kD, true)) != RTP_OK) return st;
  if ((st = check_view(k_ring, hm.n_lkv, kD, true)) != RTP_OK) return st;
  if ((st = check_view(v_ring, hm.n_lkv, kD, true)) != RTP_OK) return st;
  RingWriteParams p;
  memset(&p, 0, sizeof(p));
  p.k = static_cast<const uint16_t*>(k.ptr); p.k_sb = k.stride_b; p.k_sl = k.stride_l;
  p.v = static_cast<const uint16_t*>(v.ptr); p.v_sb = v.stride_b; p.v_sl = v.stride_l;
  p.kr = static_cast<uint16_t*>(k_ring.ptr); p.kr_sb = k_ring.stride_b; p.kr_sl = k_ring.stride_l;
  p.vr = static_cast<uint16_t*>(v_ring.ptr); p.vr_sb = v_ring.stride_b; p.vr_sl = v_ring.stride_l;
  const int64_t pos0 = shape->q_pos0, end = pos0 + shape->Lq;
  p.pos0 = pos0;
  p.a0 = pos0;
  p.a1 = std::max(pos0, std::min<int64_t>(n_sink, end));
  p.w0 = std::max<int64_t>(std::max<int64_t>(n_sink, end - window), pos0);
  p.w1 = std::max(p.w0, end);
  p.n_sink = n_sink;
  p.window = window;
  p.n_lkv = hm.n_lkv;
  for (int i = 0; i < hm.n_lkv; ++i) p.lkv[i] = hm.lkv[i];
  const int64_t items = ((p.a1 - p.a0) + (p.w1 - p.w0)) * hm.n_lkv * 16;
  if (items == 0) return RTP_OK;
  const int64_t blocks = (items + kRingThreads - 1) / kRingThreads;
  if (blocks > 0x7FFFFFFF || shape->B > 65535) return RTP_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  TraceScope tr("ring_write", s);
  ring_write_kernel<<<dim3((unsigned)blocks, shape->B), kRingThreads, 0, s>>>(p);
  return check_cuda(cudaGetLastError());
}

extern "C" rtp_status rtp_local_attn_decode_ring(const rtp_shape* shape, const uint8_t* kv_role,
                                                 int32_t window, int32_t n_sink, rtp_view q,
                                                 rtp_view k_ring, rtp_view v_ring,
                                                 float softmax_scale, rtp_view o, float* lse,
                                                 void* ws, size_t ws_bytes, rtp_stream_t stream) {
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
  if ((st = check_view(k_ring, hm.n_lkv, kD, true)) != RTP_OK) return st;
  if ((st = check_view(v_ring, hm.n_lkv, kD, true)) != RTP_OK) return st;
  if ((st = check_view(o, shape->H, kD, true)) != RTP_OK) return st;
  if (ws == nullptr || ws_bytes < kStatusBytes) return RTP_ERR_WORKSPACE_TOO_SMALL;
  return decode_range(shape, hm.lkv, hm.n_lkv, window, n_sink, q, k_ring, v_ring, softmax_scale,
                      o, lse, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream), window);
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
  return prefill_dense(shape, q, k, v, softmax_scale, o, lse, ws, s);
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
  if ((thr == nullptr) != (jtie == nullptr)) return RTP_ERR_INVALID_ARG;
  const bool all_keys = thr == nullptr;  // p >= 1: every causal key, dense tiles
  if ((st = check_view(q, shape->H, kD, true)) != RTP_OK) return st;
  if ((st = check_view(k, shape->Hkv, kD, true)) != RTP_OK) return st;
  if ((st = check_view(v, shape->Hkv, kD, true)) != RTP_OK) return st;
  if ((st = check_view(o, shape->H, kD, true)) != RTP_OK) return st;
  if ((st = check_view(q16, hm.n_ret, kR, !all_keys)) != RTP_OK) return st;
  if ((st = check_view(k16, hm.H_k16, kR, !all_keys)) != RTP_OK) return st;
  if (ws == nullptr || ws_bytes < kStatusBytes) return RTP_ERR_WORKSPACE_TOO_SMALL;
  if (all_keys)
    return prefill_dense_retrieval(shape, hm, q, k, v, softmax_scale, o, lse, ws,
                                   reinterpret_cast<cudaStream_t>(stream));
  return prefill_sparse(shape, hm, q, k, v, q16, k16, thr, jtie, softmax_scale, o, lse, ws,
                        reinterpret_cast<cudaStream_t>(stream));
}

// ====================================================================== no-allocation variant
// Scratch for rtp_local_attn_decode_noalloc: split-KV partials and merge
// counters in a file-scope device array instead of a caller workspace.
namespace rtp {
namespace {

__device__ __align__(256) unsigned char g_noalloc_scratch[RTP_NOALLOC_SCRATCH_BYTES];

// Device address of the array on the current device.  In host code the symbol
// itself is only a host-side stand-in, so the address is looked up on every
// call: a lookup allocates nothing, costs far less than the launch, and stays
// right after the context is destroyed and created again (cudaDeviceReset),
// which reloads the module at a new address.
rtp_status noalloc_scratch(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
    return RTP_ERR_CUDA;
  *out = p;
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
