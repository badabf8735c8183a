// proj.cu -- 16-dim indexer projection (rtp_index_scores).
//
// q16 = W^Q q and k16 = W^K k per retrieval head ("Low-Dimensional Projection
// Mechanism" of the paper-graph-ui summary of arXiv 2605.16928), fp32
// accumulation in a fixed order (four interleaved chains over d, then a fixed
// tree), one bf16 round-to-nearest-even.
//
// HBM-bound: each CTA stages 32 input rows (256 B each) and one 128x16 weight
// in shared memory; 4 threads per row each produce 4 of the 16 outputs.
#include <algorithm>

#include "rtp_host.h"

namespace rtp {
namespace {

constexpr int kProjRows = 32;
constexpr int kProjThreads = 128;

struct ProjJob {
  const uint16_t* x;   // [B][L][heads][128]
  int64_t x_sb, x_sl;
  const uint16_t* W;   // [slots][128][16]
  uint16_t* out;       // [B][L][slots][16]
  int64_t o_sb, o_sl;
  int L;
  int n_slots;
};

// Up to two projections (the query rows and the key rows) in one launch:
// blockIdx.y < job[0].n_slots belongs to job 0, the rest to job 1.
struct ProjParams {
  ProjJob job[2];
  int16_t head_of_slot[2][kMaxHeads];
};

__global__ void __launch_bounds__(kProjThreads) proj16_kernel(const ProjParams p) {
  __shared__ __align__(16) float sW[kD][kR];
  __shared__ float sX[kProjRows][kD + 1];
  const int jb = blockIdx.y < p.job[0].n_slots ? 0 : 1;
  const ProjJob& J = p.job[jb];
  const int slot = blockIdx.y - (jb ? p.job[0].n_slots : 0);
  const int b = blockIdx.z;
  const int row0 = blockIdx.x * kProjRows;
  if (row0 >= J.L) return;
  const int tid = threadIdx.x;
  const int nrows = min(kProjRows, J.L - row0);

  // the weight: 256 chunks of 8 bf16, two per thread
  const uint4* W = reinterpret_cast<const uint4*>(J.W + (size_t)slot * kD * kR);
  for (int c = tid; c < kD * kR / 8; c += kProjThreads) {
    const uint4 v = W[c];
    float* dst = &sW[0][0] + c * 8;
    dst[0] = bf16_lo(v.x); dst[1] = bf16_hi(v.x);
    dst[2] = bf16_lo(v.y); dst[3] = bf16_hi(v.y);
    dst[4] = bf16_lo(v.z); dst[5] = bf16_hi(v.z);
    dst[6] = bf16_lo(v.w); dst[7] = bf16_hi(v.w);
  }
  const int head = p.head_of_slot[jb][slot];
  // the rows: 16 chunks of 16 bytes each (rows past L are not read)
  for (int c = tid; c < nrows * 16; c += kProjThreads) {
    const int r = c / 16, ch = c % 16;
    const uint16_t* src = J.x + b * J.x_sb + (int64_t)(row0 + r) * J.x_sl + head * kD + ch * 8;
    const uint4 v = *reinterpret_cast<const uint4*>(src);
    float* dst = &sX[r][ch * 8];
    dst[0] = bf16_lo(v.x); dst[1] = bf16_hi(v.x);
    dst[2] = bf16_lo(v.y); dst[3] = bf16_hi(v.y);
    dst[4] = bf16_lo(v.z); dst[5] = bf16_hi(v.z);
    dst[6] = bf16_lo(v.w); dst[7] = bf16_hi(v.w);
  }
  __syncthreads();

  // thread (r, c0): outputs c0..c0+3 of row r; each is four fp32 chains over
  // d = q, q+4, q+8, ... (q = 0..3) summed as ((a0 + a1) + (a2 + a3)): a fixed
  // order shared by every call, so a key's k16 is the same in prefill and decode
  const int r = tid / 4;
  const int c0 = (tid % 4) * 4;
  if (r >= nrows) return;
  float acc[4][4];
#pragma unroll
  for (int q = 0; q < 4; ++q)
#pragma unroll
    for (int o = 0; o < 4; ++o) acc[q][o] = 0.f;
#pragma unroll 8
  for (int d = 0; d < kD; d += 4) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float xv = sX[r][d + q];
      const float4 w = *reinterpret_cast<const float4*>(&sW[d + q][c0]);
      acc[q][0] = fmaf(xv, w.x, acc[q][0]);
      acc[q][1] = fmaf(xv, w.y, acc[q][1]);
      acc[q][2] = fmaf(xv, w.z, acc[q][2]);
      acc[q][3] = fmaf(xv, w.w, acc[q][3]);
    }
  }
  float out[4];
#pragma unroll
  for (int o = 0; o < 4; ++o)
    out[o] = __fadd_rn(__fadd_rn(acc[0][o], acc[1][o]), __fadd_rn(acc[2][o], acc[3][o]));
  uint2 ov;
  ov.x = pack_bf16x2(out[0], out[1]);
  ov.y = pack_bf16x2(out[2], out[3]);
  uint16_t* dst = J.out + b * J.o_sb + (int64_t)(row0 + r) * J.o_sl + slot * kR + c0;
  *reinterpret_cast<uint2*>(dst) = ov;
}

void set_job(ProjJob& J, const rtp_view& x, int L, const void* W, int n_slots,
             const rtp_view& out) {
  J.x = static_cast<const uint16_t*>(x.ptr);
  J.x_sb = x.stride_b;
  J.x_sl = x.stride_l;
  J.W = static_cast<const uint16_t*>(W);
  J.out = static_cast<uint16_t*>(out.ptr);
  J.o_sb = out.stride_b;
  J.o_sl = out.stride_l;
  J.L = L;
  J.n_slots = n_slots;
}

}  // namespace
}  // namespace rtp

using namespace rtp;

extern "C" rtp_status rtp_index_scores(const rtp_shape* shape, const uint8_t* kv_role,
                                       int32_t k16_per_kv_head, rtp_view q, rtp_view k,
                                       const void* Wq16, const void* Wk16, rtp_view q16,
                                       rtp_view k16, rtp_stream_t stream) {
  rtp_status st = check_shape(shape);
  if (st != RTP_OK) return st;
  HeadMap hm;
  if ((st = make_headmap(shape, kv_role, k16_per_kv_head, &hm)) != RTP_OK) return st;
  const bool do_q = shape->Lq > 0 && shape->B > 0 && hm.n_ret > 0;
  const bool do_k = shape->Lk > 0 && shape->B > 0 && hm.n_ret > 0;
  if ((st = check_view(q, shape->H, kD, do_q)) != RTP_OK) return st;
  if ((st = check_view(q16, hm.n_ret, kR, do_q)) != RTP_OK) return st;
  if ((st = check_view(k, shape->Hkv, kD, do_k)) != RTP_OK) return st;
  if ((st = check_view(k16, hm.H_k16, kR, do_k)) != RTP_OK) return st;
  if (do_q && Wq16 == nullptr) return RTP_ERR_INVALID_ARG;
  if (do_k && Wk16 == nullptr) return RTP_ERR_INVALID_ARG;
  if ((do_q && !aligned16(Wq16)) || (do_k && !aligned16(Wk16))) return RTP_ERR_ALIGNMENT;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (!do_q && !do_k) return RTP_OK;
  ProjParams p;
  memset(&p, 0, sizeof(p));
  int nj = 0, max_rows = 0;
  if (do_q) {
    set_job(p.job[nj], q, shape->Lq, Wq16, hm.n_ret, q16);
    for (int sl = 0; sl < hm.n_ret; ++sl) p.head_of_slot[nj][sl] = hm.ret_q[sl];
    max_rows = std::max(max_rows, shape->Lq);
    ++nj;
  }
  if (do_k) {
    set_job(p.job[nj], k, shape->Lk, Wk16, hm.H_k16, k16);
    for (int sl = 0; sl < hm.H_k16; ++sl)
      p.head_of_slot[nj][sl] = k16_per_kv_head ? hm.rkv[sl] : (int16_t)(hm.ret_q[sl] / hm.G);
    max_rows = std::max(max_rows, shape->Lk);
    ++nj;
  }
  dim3 grid((max_rows + kProjRows - 1) / kProjRows, p.job[0].n_slots + p.job[1].n_slots, shape->B);
  if (grid.z > 65535 || grid.y > 65535) return RTP_ERR_UNSUPPORTED;
  TraceScope tr("proj16", s);
  proj16_kernel<<<grid, kProjThreads, 0, s>>>(p);
  st = check_cuda(cudaGetLastError());
  return st;
}
