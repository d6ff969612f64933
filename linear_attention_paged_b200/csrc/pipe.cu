// pipe.cu -- a decode-step pipeline over host buffers: the inputs of step k+1 are
// uploaded and the output of step k-1 downloaded while step k computes.
//
// Two device sets of (q, gate, out) alternate between steps.  Step k uses set
// b = k % 2:
//   upload stream    waits until step k-2 has finished reading set b, copies q and
//                    gate from the host into set b, records up[b];
//   compute stream   waits for up[b] and for step k-2's output copy (down[b]), runs
//                    wa_hsa_step on set b, records done[b];
//   download stream  waits for done[b], copies out from set b to the host, records
//                    down[b].
// Host-to-device and device-to-host copies use separate streams so that both
// overlap the compute stream (PCIe is full duplex).  The caller keeps each host
// buffer untouched (inputs) or unread (output) until wa_pipe_sync returns or a
// later wa_pipe_end is ordered before its own reads.
#include <cuda_runtime.h>

#include <cstring>

#include "wa_internal.h"

struct wa_pipe {
  wa_step_args args{};
  void* q[2] = {nullptr, nullptr};
  const float* gate[2] = {nullptr, nullptr};
  void* out[2] = {nullptr, nullptr};
  void* ws = nullptr;
  size_t ws_bytes = 0;
  size_t q_bytes = 0, gate_bytes = 0, out_bytes = 0;
  cudaStream_t comp = nullptr, up_s = nullptr, down_s = nullptr;
  cudaEvent_t up[2] = {nullptr, nullptr}, done[2] = {nullptr, nullptr}, down[2] = {nullptr, nullptr};
  cudaEvent_t mark = nullptr;
  long long n = 0;
};

namespace {
using wa::set_error;
wa_status ok_or(cudaError_t e, const char* what) {
  return e == cudaSuccess ? WA_OK : set_error(WA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}
#define PIPE_TRY(expr, what)                       \
  do {                                             \
    const wa_status s_ = ok_or((expr), (what));    \
    if (s_ != WA_OK) return s_;                    \
  } while (0)
}  // namespace

extern "C" {

wa_status wa_pipe_create(const wa_step_args* a, void* q1, const float* gate1, void* out1, void* ws,
                         size_t ws_bytes, void* stream, wa_pipe** out) {
  if (!out) return set_error(WA_ERR_INVALID_ARG, "NULL output");
  *out = nullptr;
  if (!a || !a->q || !a->gate || !a->out || !q1 || !gate1 || !out1 || !ws)
    return set_error(WA_ERR_INVALID_ARG, "NULL pointer");
  if (a->Nq < 1 || a->H < 1 || a->d < 1) return set_error(WA_ERR_INVALID_ARG, "bad sizes");
  const size_t need = wa_hsa_step_workspace_size(a);
  if (need == 0) return WA_ERR_INVALID_ARG;          // the reason is already set
  if (ws_bytes < need) return set_error(WA_ERR_WORKSPACE, "workspace %zu bytes, need %zu", ws_bytes, need);
  wa_pipe* p = new wa_pipe;
  std::memcpy(&p->args, a, sizeof(wa_step_args));
  p->q[0] = const_cast<void*>(a->q); p->q[1] = q1;
  p->gate[0] = a->gate; p->gate[1] = gate1;
  p->out[0] = a->out; p->out[1] = out1;
  p->ws = ws; p->ws_bytes = ws_bytes;
  const size_t es = a->dtype == WA_BF16 ? 2 : 4;
  p->q_bytes = static_cast<size_t>(a->Nq) * a->H * a->d * es;
  p->out_bytes = p->q_bytes;
  p->gate_bytes = static_cast<size_t>(a->Nq) * a->H * sizeof(float);
  p->comp = static_cast<cudaStream_t>(stream);
  bool ok = cudaStreamCreateWithFlags(&p->up_s, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&p->down_s, cudaStreamNonBlocking) == cudaSuccess &&
            cudaEventCreateWithFlags(&p->mark, cudaEventDisableTiming) == cudaSuccess;
  for (int b = 0; ok && b < 2; ++b)
    ok = cudaEventCreateWithFlags(&p->up[b], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&p->done[b], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&p->down[b], cudaEventDisableTiming) == cudaSuccess;
  if (!ok) {
    wa_pipe_destroy(p);
    return set_error(WA_ERR_CUDA, "could not create the pipeline's streams and events");
  }
  *out = p;
  return WA_OK;
}

wa_status wa_pipe_destroy(wa_pipe* p) {
  if (!p) return WA_OK;
  if (p->up_s) cudaStreamSynchronize(p->up_s);
  if (p->down_s) cudaStreamSynchronize(p->down_s);
  for (int b = 0; b < 2; ++b) {
    if (p->up[b]) cudaEventDestroy(p->up[b]);
    if (p->done[b]) cudaEventDestroy(p->done[b]);
    if (p->down[b]) cudaEventDestroy(p->down[b]);
  }
  if (p->mark) cudaEventDestroy(p->mark);
  if (p->up_s) cudaStreamDestroy(p->up_s);
  if (p->down_s) cudaStreamDestroy(p->down_s);
  delete p;
  return WA_OK;
}

wa_status wa_pipe_begin(wa_pipe* p) {
  if (!p) return set_error(WA_ERR_INVALID_ARG, "NULL pipeline");
  PIPE_TRY(cudaEventRecord(p->mark, p->comp), "event record");
  PIPE_TRY(cudaStreamWaitEvent(p->up_s, p->mark, 0), "stream wait");
  PIPE_TRY(cudaStreamWaitEvent(p->down_s, p->mark, 0), "stream wait");
  return WA_OK;
}

wa_status wa_pipe_submit(wa_pipe* p, const void* q_host, const float* gate_host, void* out_host) {
  if (!p || !q_host || !gate_host || !out_host) return set_error(WA_ERR_INVALID_ARG, "NULL pointer");
  const int b = static_cast<int>(p->n & 1);
  if (p->n >= 2) PIPE_TRY(cudaStreamWaitEvent(p->up_s, p->done[b], 0), "stream wait");
  PIPE_TRY(cudaMemcpyAsync(p->q[b], q_host, p->q_bytes, cudaMemcpyHostToDevice, p->up_s), "upload q");
  PIPE_TRY(cudaMemcpyAsync(const_cast<float*>(p->gate[b]), gate_host, p->gate_bytes,
                           cudaMemcpyHostToDevice, p->up_s), "upload gate");
  PIPE_TRY(cudaEventRecord(p->up[b], p->up_s), "event record");
  PIPE_TRY(cudaStreamWaitEvent(p->comp, p->up[b], 0), "stream wait");
  if (p->n >= 2) PIPE_TRY(cudaStreamWaitEvent(p->comp, p->down[b], 0), "stream wait");
  p->args.q = p->q[b];
  p->args.gate = p->gate[b];
  p->args.out = p->out[b];
  const wa_status s = wa_hsa_step(&p->args, p->ws, p->ws_bytes, p->comp);
  if (s != WA_OK) return s;
  PIPE_TRY(cudaEventRecord(p->done[b], p->comp), "event record");
  PIPE_TRY(cudaStreamWaitEvent(p->down_s, p->done[b], 0), "stream wait");
  PIPE_TRY(cudaMemcpyAsync(out_host, p->out[b], p->out_bytes, cudaMemcpyDeviceToHost, p->down_s),
           "download out");
  PIPE_TRY(cudaEventRecord(p->down[b], p->down_s), "event record");
  ++p->n;
  return WA_OK;
}

wa_status wa_pipe_end(wa_pipe* p) {
  if (!p) return set_error(WA_ERR_INVALID_ARG, "NULL pipeline");
  PIPE_TRY(cudaEventRecord(p->mark, p->up_s), "event record");
  PIPE_TRY(cudaStreamWaitEvent(p->comp, p->mark, 0), "stream wait");
  PIPE_TRY(cudaEventRecord(p->mark, p->down_s), "event record");
  PIPE_TRY(cudaStreamWaitEvent(p->comp, p->mark, 0), "stream wait");
  return WA_OK;
}

wa_status wa_pipe_sync(wa_pipe* p) {
  if (!p) return set_error(WA_ERR_INVALID_ARG, "NULL pipeline");
  PIPE_TRY(cudaStreamSynchronize(p->up_s), "synchronize");
  PIPE_TRY(cudaStreamSynchronize(p->comp), "synchronize");
  PIPE_TRY(cudaStreamSynchronize(p->down_s), "synchronize");
  return WA_OK;
}

}  // extern "C"
