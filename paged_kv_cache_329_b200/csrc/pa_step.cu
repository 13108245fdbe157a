// A decode step captured once as a CUDA graph and replayed (pa_step_* in pa.h).
//
// The step is the serving loop's unit of work on the pages' cache ("vllm" 2.2 Decode: every step
// appends the new token's K,V and attends over the cache; "PagedAttention原理", "解决COW": shared
// blocks are copied before they are written): host->device copies of the step's inputs, the
// copy-on-write block copies, the slot-mapped write, the paged decode, and the device->host copy
// of the output.  Replaying one graph replaces a dozen stream operations per step.
#include <cuda_runtime.h>

#include <algorithm>
#include <new>
#include <vector>

#include "pa_internal.h"

namespace {

struct Copy {
  void* dst;
  const void* src;
  size_t bytes;
};

}  // namespace

struct pa_step {
  cudaGraph_t graph = nullptr;             // H2D, kernels, D2H: pa_step_run / pa_step_launch
  cudaGraphExec_t exec = nullptr;
  cudaGraph_t kgraph = nullptr;            // kernels only: pa_step_launch_async
  cudaGraphExec_t kexec = nullptr;
  std::vector<Copy> h2d;                   // the merged input copies
  cudaStream_t s_in = nullptr, s_out = nullptr;
  cudaEvent_t ev_in = nullptr, ev_done = nullptr, ev_out = nullptr;
  pa_step_desc desc;
};

namespace {

bool pinned(const void* p) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return at.type == cudaMemoryTypeHost;
}

// The step's input copies, merged where host and device buffers keep the same relative placement.
std::vector<Copy> input_copies(const pa_step_desc& d) {
  const size_t es = pa::elem_size(d.kv_dtype);
  const size_t q_bytes = static_cast<size_t>(d.S) * d.H * d.d * es;
  const size_t kv_bytes = static_cast<size_t>(d.S) * d.Hk * d.d * es;
  const size_t tbl_bytes = static_cast<size_t>(d.S) * d.max_blocks_per_seq * sizeof(int32_t);
  const Copy h2d[] = {
      {d.d_query, d.h_query, q_bytes},
      {d.d_key, d.h_key, kv_bytes},
      {d.d_value, d.h_value, kv_bytes},
      {d.d_slots, d.h_slots, static_cast<size_t>(d.S) * sizeof(int64_t)},
      {d.d_pairs, d.h_pairs, static_cast<size_t>(d.max_pairs) * 2 * sizeof(int32_t)},
      {d.d_pairs + 2 * static_cast<size_t>(d.max_pairs), d.h_n_pairs, sizeof(int32_t)},
      {d.d_tables, d.h_tables, tbl_bytes},
      {d.d_lens, d.h_lens, static_cast<size_t>(d.S) * sizeof(int32_t)},
  };
  // Copies whose host and device buffers keep the same relative placement (e.g. carved from one
  // host block and one device block with equal offsets) are merged into one transfer, gaps of at
  // most 4 KiB included.
  std::vector<Copy> list;
  for (const Copy& c : h2d)
    if (c.bytes) list.push_back(c);
  std::sort(list.begin(), list.end(), [](const Copy& x, const Copy& y) { return x.src < y.src; });
  std::vector<Copy> merged;
  for (const Copy& c : list) {
    if (!merged.empty()) {
      Copy& m = merged.back();
      const char* m_src = static_cast<const char*>(m.src);
      const char* c_src = static_cast<const char*>(c.src);
      const char* m_dst = static_cast<const char*>(m.dst);
      const char* c_dst = static_cast<const char*>(c.dst);
      if (c_src >= m_src + m.bytes && c_src - m_src == c_dst - m_dst && c_src - (m_src + m.bytes) <= 4096) {
        m.bytes = static_cast<size_t>(c_src - m_src) + c.bytes;
        continue;
      }
    }
    merged.push_back(c);
  }
  return merged;
}

// copy-on-write copies, cache write, decode (pa_decode_step: the copies, the writes and the plan in
// one kernel, the pair count read on the device)
pa_status record_kernels(const pa_step_desc& d, cudaStream_t s) {
  if (d.max_pairs > pa::kMaxStepPairs) {  // too many pairs for the fused form: three calls in order
    pa_status st = pa::copy_blocks_counted(d.k_cache, d.v_cache, d.d_pairs,
                                           d.d_pairs + 2 * static_cast<size_t>(d.max_pairs), d.max_pairs, d.Hk, d.d,
                                           d.B, d.n_blocks, d.kv_dtype, s);
    if (st == PA_OK)
      st = pa_cache_write(d.k_cache, d.v_cache, d.d_key, d.d_value, d.d_slots, d.S, d.Hk, d.d, d.B, d.n_blocks,
                          d.kv_dtype, s);
    if (st == PA_OK)
      st = pa_decode(d.d_out, d.out_dtype, d.d_query, d.k_cache, d.v_cache, d.d_tables, d.d_lens, d.S, d.H, d.Hk,
                     d.d, d.B, d.n_blocks, d.max_blocks_per_seq, d.max_context_len, d.scale, d.kv_dtype,
                     d.partition_size, d.workspace, d.workspace_bytes, s);
    return st;
  }
  return pa_decode_step(d.d_out, d.out_dtype, d.d_query, d.k_cache, d.v_cache, d.d_tables, d.d_lens, d.d_key,
                        d.d_value, d.d_slots, d.S, d.d_pairs, d.d_pairs + 2 * static_cast<size_t>(d.max_pairs),
                        d.max_pairs, d.S, d.H, d.Hk, d.d, d.B, d.n_blocks, d.max_blocks_per_seq, d.max_context_len,
                        d.scale, d.kv_dtype, d.partition_size, d.workspace, d.workspace_bytes, s);
}

size_t out_bytes(const pa_step_desc& d) {
  return static_cast<size_t>(d.S) * d.H * d.d * pa::elem_size(d.out_dtype);
}

pa_status record(const pa_step_desc& d, cudaStream_t s) {
  for (const Copy& c : input_copies(d)) {
    const cudaError_t e = cudaMemcpyAsync(c.dst, c.src, c.bytes, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, "pa_step_create: capture of a copy failed: %s", cudaGetErrorString(e));
  }
  const pa_status st = record_kernels(d, s);
  if (st != PA_OK) return st;
  const cudaError_t e = cudaMemcpyAsync(d.h_out, d.d_out, out_bytes(d), cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, "pa_step_create: capture of the output copy failed: %s", cudaGetErrorString(e));
  return PA_OK;
}

// Captures `rec` on a private stream and instantiates it.
template <class Rec>
pa_status capture(const pa_step_desc& d, Rec rec, cudaGraph_t* graph, cudaGraphExec_t* exec) {
  cudaStream_t s = nullptr;
  cudaError_t e = cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking);
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, "pa_step_create: %s", cudaGetErrorString(e));
  e = cudaStreamBeginCapture(s, cudaStreamCaptureModeRelaxed);
  pa_status st = e == cudaSuccess ? rec(d, s) : pa::fail(PA_ERR_CUDA, "pa_step_create: %s", cudaGetErrorString(e));
  if (e == cudaSuccess) {
    const cudaError_t e2 = cudaStreamEndCapture(s, graph);  // always end the capture
    if (st == PA_OK && e2 != cudaSuccess) st = pa::fail(PA_ERR_CUDA, "pa_step_create: %s", cudaGetErrorString(e2));
  }
  if (st == PA_OK) {
    e = cudaGraphInstantiate(exec, *graph, 0);
    if (e != cudaSuccess) st = pa::fail(PA_ERR_CUDA, "pa_step_create: instantiate: %s", cudaGetErrorString(e));
  }
  cudaStreamDestroy(s);
  return st;
}

}  // namespace

extern "C" pa_step* pa_step_create(const pa_step_desc* desc) {
  if (!desc) {
    pa::fail(PA_ERR_INVALID_ARG, "pa_step_create: null descriptor");
    return nullptr;
  }
  const pa_step_desc& d = *desc;
  const void* host[] = {d.h_query, d.h_key, d.h_value, d.h_slots, d.h_pairs, d.h_n_pairs, d.h_tables, d.h_lens, d.h_out};
  for (const void* p : host)
    if (!p || !pinned(p)) {
      pa::fail(PA_ERR_INVALID_ARG, "pa_step_create: every host buffer must be non-null pinned memory");
      return nullptr;
    }
  if (d.S <= 0 || d.max_pairs < 0 || !d.d_pairs || !d.d_query || !d.d_key || !d.d_value || !d.d_slots || !d.d_tables ||
      !d.d_lens || !d.d_out) {
    pa::fail(PA_ERR_INVALID_ARG, "pa_step_create: bad sizes or null device buffer");
    return nullptr;
  }
  pa_step* step = new (std::nothrow) pa_step;
  if (!step) {
    pa::fail(PA_ERR_INVALID_ARG, "pa_step_create: out of host memory");
    return nullptr;
  }
  step->desc = d;
  pa_status st = capture(d, record, &step->graph, &step->exec);
  if (st == PA_OK) st = capture(d, record_kernels, &step->kgraph, &step->kexec);
  if (st == PA_OK) {
    step->h2d = input_copies(d);
    cudaError_t e = cudaStreamCreateWithFlags(&step->s_in, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&step->s_out, cudaStreamNonBlocking);
    for (cudaEvent_t* ev : {&step->ev_in, &step->ev_done, &step->ev_out})
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
    if (e != cudaSuccess) st = pa::fail(PA_ERR_CUDA, "pa_step_create: %s", cudaGetErrorString(e));
  }
  if (st != PA_OK) {
    pa_step_destroy(step);
    return nullptr;
  }
  pa::ok();
  return step;
}

extern "C" pa_status pa_step_run(pa_step* step, void* stream) {
  if (!step || !step->exec) return pa::fail(PA_ERR_INVALID_ARG, "pa_step_run: null step");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaGraphLaunch(step->exec, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, "pa_step_run: %s", cudaGetErrorString(e));
  return pa::ok();
}

extern "C" pa_status pa_step_launch(pa_step* step, void* stream) {
  if (!step || !step->exec) return pa::fail(PA_ERR_INVALID_ARG, "pa_step_launch: null step");
  const cudaError_t e = cudaGraphLaunch(step->exec, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, "pa_step_launch: %s", cudaGetErrorString(e));
  return pa::ok();
}

extern "C" pa_status pa_step_launch_async(pa_step* step, void* stream) {
  if (!step || !step->kexec) return pa::fail(PA_ERR_INVALID_ARG, "pa_step_launch_async: null step");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const pa_step_desc& d = step->desc;
  // inputs: once this step's previous kernels no longer read its device inputs
  cudaError_t e = cudaStreamWaitEvent(step->s_in, step->ev_done, 0);
  for (size_t i = 0; e == cudaSuccess && i < step->h2d.size(); ++i) {
    const Copy& c = step->h2d[i];
    e = cudaMemcpyAsync(c.dst, c.src, c.bytes, cudaMemcpyHostToDevice, step->s_in);
  }
  if (e == cudaSuccess) e = cudaEventRecord(step->ev_in, step->s_in);
  // kernels: after the inputs, and after this step's previous output copy has left d_out
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s, step->ev_in, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s, step->ev_out, 0);
  if (e == cudaSuccess) e = cudaGraphLaunch(step->kexec, s);
  if (e == cudaSuccess) e = cudaEventRecord(step->ev_done, s);
  // output
  if (e == cudaSuccess) e = cudaStreamWaitEvent(step->s_out, step->ev_done, 0);
  if (e == cudaSuccess) e = cudaMemcpyAsync(d.h_out, d.d_out, out_bytes(d), cudaMemcpyDeviceToHost, step->s_out);
  if (e == cudaSuccess) e = cudaEventRecord(step->ev_out, step->s_out);
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, "pa_step_launch_async: %s", cudaGetErrorString(e));
  return pa::ok();
}

extern "C" pa_status pa_step_wait(pa_step* step) {
  if (!step || !step->ev_out) return pa::fail(PA_ERR_INVALID_ARG, "pa_step_wait: null step");
  const cudaError_t e = cudaEventSynchronize(step->ev_out);
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, "pa_step_wait: %s", cudaGetErrorString(e));
  return pa::ok();
}

extern "C" void pa_step_destroy(pa_step* step) {
  if (!step) return;
  for (cudaStream_t s : {step->s_in, step->s_out})
    if (s) {
      cudaStreamSynchronize(s);
      cudaStreamDestroy(s);
    }
  for (cudaEvent_t ev : {step->ev_in, step->ev_done, step->ev_out})
    if (ev) cudaEventDestroy(ev);
  if (step->kexec) cudaGraphExecDestroy(step->kexec);
  if (step->kgraph) cudaGraphDestroy(step->kgraph);
  if (step->exec) cudaGraphExecDestroy(step->exec);
  if (step->graph) cudaGraphDestroy(step->graph);
  delete step;
}
