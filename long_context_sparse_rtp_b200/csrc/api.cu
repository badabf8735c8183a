// api.cu -- status strings, version, workspace initialisation and the device
// status word shared by every entry point.
#include <mutex>
#include <string>
#include <vector>

#include "rtp_host.h"

using namespace rtp;

extern "C" const char* rtp_status_string(rtp_status status) {
  switch (status) {
    case RTP_OK: return "RTP_OK";
    case RTP_ERR_INVALID_ARG: return "RTP_ERR_INVALID_ARG";
    case RTP_ERR_UNSUPPORTED: return "RTP_ERR_UNSUPPORTED";
    case RTP_ERR_ALIGNMENT: return "RTP_ERR_ALIGNMENT";
    case RTP_ERR_WORKSPACE_TOO_SMALL: return "RTP_ERR_WORKSPACE_TOO_SMALL";
    case RTP_ERR_CUDA: return "RTP_ERR_CUDA";
    case RTP_ERR_DEVICE_TIMEOUT: return "RTP_ERR_DEVICE_TIMEOUT";
    case RTP_ERR_SCRATCH_LIMIT: return "RTP_ERR_SCRATCH_LIMIT";
  }
  return "RTP_ERR_UNKNOWN";
}

extern "C" const char* rtp_version(void) { return "0.1.0"; }

extern "C" rtp_status rtp_workspace_init(void* ws, size_t ws_bytes, rtp_stream_t stream) {
  if (ws == nullptr || ws_bytes < kStatusBytes) return RTP_ERR_WORKSPACE_TOO_SMALL;
  if (!aligned16(ws)) return RTP_ERR_ALIGNMENT;
  return check_cuda(cudaMemsetAsync(ws, 0, ws_bytes, reinterpret_cast<cudaStream_t>(stream)));
}

extern "C" rtp_status rtp_get_device_status(void* ws, rtp_stream_t stream) {
  if (ws == nullptr) return RTP_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  DevStatus host;
  if (cudaMemcpyAsync(&host, ws, sizeof(host), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return RTP_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return RTP_ERR_CUDA;
  if (host.code == 0) return RTP_OK;
  const int32_t zero = 0;
  if (cudaMemcpyAsync(ws, &zero, sizeof(zero), cudaMemcpyHostToDevice, s) != cudaSuccess)
    return RTP_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return RTP_ERR_CUDA;
  return (rtp_status)host.code;
}

// ---------------------------------------------------------------- kernel trace
namespace rtp {
namespace {
struct TraceRec {
  std::string name;
  cudaEvent_t start, stop;
};
std::mutex g_trace_mu;
bool g_trace_on = false;
std::vector<TraceRec> g_trace;       // completed or in-flight launches
std::vector<cudaEvent_t> g_free;     // recycled events
thread_local int g_open = -1;        // index of the launch being bracketed

cudaEvent_t take_event() {
  if (!g_free.empty()) {
    cudaEvent_t e = g_free.back();
    g_free.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}
}  // namespace

// Under stream capture the events become event-record nodes of the graph
// (external records), so every replay of the graph times its kernels again.
void record(cudaEvent_t e, cudaStream_t s) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags(e, s, cudaEventRecordExternal);
  else
    cudaEventRecord(e, s);
}

void trace_begin(const char* name, cudaStream_t s) {
  if (!g_trace_on) return;
  std::lock_guard<std::mutex> lk(g_trace_mu);
  TraceRec r{name, take_event(), take_event()};
  record(r.start, s);
  g_trace.push_back(r);
  g_open = (int)g_trace.size() - 1;
}

void trace_end(cudaStream_t s) {
  if (!g_trace_on || g_open < 0) return;
  std::lock_guard<std::mutex> lk(g_trace_mu);
  if (g_open < (int)g_trace.size()) record(g_trace[g_open].stop, s);
  g_open = -1;
}
}  // namespace rtp

extern "C" void rtp_trace_enable(int on) {
  rtp::g_trace_on = on != 0;
  if (on) {  // keep a few events ready so that a capture does not have to create them
    std::lock_guard<std::mutex> lk(rtp::g_trace_mu);
    while (rtp::g_free.size() < 64) {
      cudaEvent_t e = nullptr;
      if (cudaEventCreate(&e) != cudaSuccess) break;
      rtp::g_free.push_back(e);
    }
  }
}

extern "C" void rtp_trace_reset(void) {
  std::lock_guard<std::mutex> lk(rtp::g_trace_mu);
  for (auto& r : rtp::g_trace) {
    rtp::g_free.push_back(r.start);
    rtp::g_free.push_back(r.stop);
  }
  rtp::g_trace.clear();
}

extern "C" int rtp_trace_timeline(rtp_trace_launch* out, int max_entries) {
  std::lock_guard<std::mutex> lk(rtp::g_trace_mu);
  if (rtp::g_trace.empty()) return 0;
  const cudaEvent_t t0 = rtp::g_trace.front().start;
  int n = 0;
  for (auto& r : rtp::g_trace) {
    if (n >= max_entries) break;
    if (cudaEventSynchronize(r.stop) != cudaSuccess) return -1;
    float a = 0.f, b = 0.f;
    if (cudaEventElapsedTime(&a, t0, r.start) != cudaSuccess ||
        cudaEventElapsedTime(&b, t0, r.stop) != cudaSuccess)
      return -1;
    memset(&out[n], 0, sizeof(out[n]));
    strncpy(out[n].name, r.name.c_str(), sizeof(out[n].name) - 1);
    out[n].start_ms = a;
    out[n].end_ms = b;
    ++n;
  }
  return n;
}

extern "C" int rtp_trace_read(rtp_trace_entry* out, int max_entries) {
  std::lock_guard<std::mutex> lk(rtp::g_trace_mu);
  int n = 0;
  for (auto& r : rtp::g_trace) {
    if (cudaEventSynchronize(r.stop) != cudaSuccess) return -1;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, r.start, r.stop) != cudaSuccess) return -1;
    int k = 0;
    while (k < n && strncmp(out[k].name, r.name.c_str(), sizeof(out[k].name)) != 0) ++k;
    if (k == n) {
      if (n >= max_entries) continue;
      memset(&out[n], 0, sizeof(out[n]));
      strncpy(out[n].name, r.name.c_str(), sizeof(out[n].name) - 1);
      ++n;
    }
    out[k].launches += 1;
    out[k].total_ms += ms;
  }
  return n;
}

// ---------------------------------------------------------------- tensor maps
#include <cudaTypedefs.h>

#include "tma.cuh"

namespace rtp {
bool tma_encode_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                     const uint64_t* strides_bytes, const uint32_t* box, int swizzle_bytes) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (encode == nullptr || rank < 1 || rank > 5) return false;
  CUtensorMapSwizzle swz;
  switch (swizzle_bytes) {
    case 0: swz = CU_TENSOR_MAP_SWIZZLE_NONE; break;
    case 32: swz = CU_TENSOR_MAP_SWIZZLE_32B; break;
    case 64: swz = CU_TENSOR_MAP_SWIZZLE_64B; break;
    case 128: swz = CU_TENSOR_MAP_SWIZZLE_128B; break;
    default: return false;
  }
  cuuint64_t d[5], st[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
    if (i > 0) st[i - 1] = strides_bytes[i - 1];
  }
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(base),
                d, st, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}
}  // namespace rtp
