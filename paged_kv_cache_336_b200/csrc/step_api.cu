// pa_decode_step: one whole decode step from host buffers (see
// include/pagedkv.h). Host code only: the block manager step, the uploads,
// the existing kernel entry points and the download, in one C call.
#include <cuda_runtime.h>

#include <cstdint>

#include "pa_internal.h"

using pagedkv::fail;
using pagedkv::ok;

namespace {

size_t elt(pa_dtype_t dt) { return dt == PA_F32 ? 4 : 2; }

size_t q_bytes(const pa_step_buffers_t* b, int n) {
  return static_cast<size_t>(n) * b->num_q_heads * b->head_dim * elt(b->dtype);
}

size_t kv_bytes(const pa_step_buffers_t* b, int n) {
  return static_cast<size_t>(n) * b->num_kv_heads * b->head_dim * elt(b->dtype);
}

// The four small staging arrays of a set, laid out back to back (host and
// device alike): slots int64 [max_seqs] | pairs int64 [max_seqs][2] |
// lengths int32 [max_seqs] | tables int32 [max_seqs][max_blocks_per_seq].
// Then one copy carries them all.
bool packed_layout(const pa_step_buffers_t* b) {
  const int m = b->max_seqs;
  return b->h_pairs == b->h_slots + m && b->d_pairs == b->d_slots + m &&
         b->h_context_lens == reinterpret_cast<int32_t*>(b->h_pairs + 2 * m) &&
         b->d_context_lens == reinterpret_cast<int32_t*>(b->d_pairs + 2 * m) &&
         b->h_tables == b->h_context_lens + m && b->d_tables == b->d_context_lens + m;
}

// Bytes of the one packed copy for n sequences: everything before the tables
// plus n table rows.
size_t packed_bytes(const pa_step_buffers_t* b, int n) {
  return static_cast<size_t>(b->max_seqs) * (8 + 16 + 4) +
         static_cast<size_t>(n) * b->max_blocks_per_seq * 4;
}

pa_status_t cuda_check(cudaError_t err, const char* what) {
  if (err != cudaSuccess) return fail(PA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(err));
  return PA_OK;
}

}  // namespace

extern "C" {

size_t pa_decode_step_h2d_bytes(const pa_step_buffers_t* b, int n, int num_copies) {
  if (b == nullptr || n < 0) return 0;
  if (packed_layout(b)) return q_bytes(b, n) + 2 * kv_bytes(b, n) + packed_bytes(b, n);
  return q_bytes(b, n) + 2 * kv_bytes(b, n) + static_cast<size_t>(n) * 8 +
         static_cast<size_t>(n) * b->max_blocks_per_seq * 4 + static_cast<size_t>(n) * 4 +
         static_cast<size_t>(num_copies) * 16;
}

size_t pa_decode_step_d2h_bytes(const pa_step_buffers_t* b, int n) {
  if (b == nullptr || n < 0) return 0;
  return q_bytes(b, n);
}

pa_status_t pa_decode_step(pa_bm_t bm, const pa_step_buffers_t* b, const int64_t* seq_ids, int n,
                           const void* q_host, const void* k_new_host, const void* v_new_host,
                           void* out_host, int* num_copies, int synchronize, uint32_t* dev_err,
                           void* stream_ptr) {
  PA_NVTX_RANGE("pa_decode_step");
  if (bm == nullptr || b == nullptr) return fail(PA_ERR_INVALID_ARG, "bm or buffers is NULL");
  if (n < 0 || n > b->max_seqs) return fail(PA_ERR_INVALID_ARG, "n=%d outside [0, max_seqs=%d]", n, b->max_seqs);
  if (num_copies) *num_copies = 0;
  if (n == 0) return ok();
  if (seq_ids == nullptr || q_host == nullptr || k_new_host == nullptr || v_new_host == nullptr ||
      out_host == nullptr)
    return fail(PA_ERR_INVALID_ARG, "NULL host buffer");
  if (b->d_q == nullptr || b->d_k_new == nullptr || b->d_v_new == nullptr || b->d_out == nullptr ||
      b->d_slots == nullptr || b->d_pairs == nullptr || b->d_tables == nullptr ||
      b->d_context_lens == nullptr || b->h_slots == nullptr || b->h_pairs == nullptr ||
      b->h_tables == nullptr || b->h_context_lens == nullptr)
    return fail(PA_ERR_INVALID_ARG, "NULL staging buffer");
  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  const bool piped = b->copy_stream != nullptr;
  if (piped && (b->upload_done == nullptr || b->compute_done == nullptr || b->download_done == nullptr ||
                b->download_stream == nullptr))
    return fail(PA_ERR_INVALID_ARG, "copy_stream set without its events and download stream");
  cudaStream_t cs = piped ? static_cast<cudaStream_t>(b->copy_stream) : stream;
  cudaStream_t ds = piped ? static_cast<cudaStream_t>(b->download_stream) : stream;
  cudaEvent_t upload_done = static_cast<cudaEvent_t>(b->upload_done);
  cudaEvent_t compute_done = static_cast<cudaEvent_t>(b->compute_done);
  cudaEvent_t download_done = static_cast<cudaEvent_t>(b->download_done);

  // 0. this set's host staging is rewritten below: its previous uploads
  // must have read it
  pa_status_t st;
  if (upload_done != nullptr &&
      (st = cuda_check(cudaEventSynchronize(upload_done), "wait for previous uploads")) != PA_OK)
    return st;

  // 1. block manager: one slot per sequence, copies where a tail is shared
  int ncow = 0;
  st = pa_bm_append_slots(bm, seq_ids, n, b->h_slots, b->h_pairs, &ncow);
  if (st != PA_OK) return st;
  st = pa_bm_export(bm, seq_ids, n, b->h_tables, b->h_context_lens, -1);
  if (st != PA_OK) return st;
  if (num_copies) *num_copies = ncow;

  // 2. uploads (on the copy stream once this set's device staging is no longer
  // used by its previous step: download_done follows that step's decode and
  // download; waiting on a never-recorded event returns at once)
  if (piped && (st = cuda_check(cudaStreamWaitEvent(cs, download_done, 0), "order uploads")) != PA_OK)
    return st;
  if ((st = cuda_check(cudaMemcpyAsync(b->d_q, q_host, q_bytes(b, n), cudaMemcpyHostToDevice, cs), "upload q")) != PA_OK) return st;
  if ((st = cuda_check(cudaMemcpyAsync(b->d_k_new, k_new_host, kv_bytes(b, n), cudaMemcpyHostToDevice, cs), "upload k_new")) != PA_OK) return st;
  if ((st = cuda_check(cudaMemcpyAsync(b->d_v_new, v_new_host, kv_bytes(b, n), cudaMemcpyHostToDevice, cs), "upload v_new")) != PA_OK) return st;
  if (packed_layout(b)) {
    if ((st = cuda_check(cudaMemcpyAsync(b->d_slots, b->h_slots, packed_bytes(b, n), cudaMemcpyHostToDevice, cs), "upload slots, pairs, lengths, tables")) != PA_OK) return st;
  } else {
    if ((st = cuda_check(cudaMemcpyAsync(b->d_slots, b->h_slots, static_cast<size_t>(n) * 8, cudaMemcpyHostToDevice, cs), "upload slots")) != PA_OK) return st;
    if ((st = cuda_check(cudaMemcpyAsync(b->d_tables, b->h_tables, static_cast<size_t>(n) * b->max_blocks_per_seq * 4, cudaMemcpyHostToDevice, cs), "upload tables")) != PA_OK) return st;
    if ((st = cuda_check(cudaMemcpyAsync(b->d_context_lens, b->h_context_lens, static_cast<size_t>(n) * 4, cudaMemcpyHostToDevice, cs), "upload lengths")) != PA_OK) return st;
    if (ncow > 0 &&
        (st = cuda_check(cudaMemcpyAsync(b->d_pairs, b->h_pairs, static_cast<size_t>(ncow) * 16, cudaMemcpyHostToDevice, cs), "upload copy pairs")) != PA_OK)
      return st;
  }

  if (piped) {
    if ((st = cuda_check(cudaEventRecord(upload_done, cs), "record uploads")) != PA_OK) return st;
    if ((st = cuda_check(cudaStreamWaitEvent(stream, upload_done, 0), "order uploads")) != PA_OK) return st;
  } else if (upload_done != nullptr) {
    if ((st = cuda_check(cudaEventRecord(upload_done, stream), "record uploads")) != PA_OK) return st;
  }

  // 3. kernels: copy-on-write copies before the append writes into them
  const size_t block_bytes = static_cast<size_t>(b->num_kv_heads) * b->block_size * b->head_dim * elt(b->dtype);
  if (ncow > 0) {
    st = pa_copy_blocks(b->k_pool, b->v_pool, b->d_pairs, ncow, block_bytes, b->num_blocks, dev_err, stream);
    if (st != PA_OK) return st;
  }
  st = pa_kv_append(b->d_k_new, b->d_v_new, b->d_slots, n, b->num_kv_heads, b->head_dim, b->block_size,
                    b->num_blocks, b->dtype, b->k_pool, b->v_pool, dev_err, stream);
  if (st != PA_OK) return st;
  st = pa_decode_split(b->d_q, b->k_pool, b->v_pool, b->d_tables, b->d_context_lens, n, b->num_q_heads,
                       b->num_kv_heads, b->head_dim, b->block_size, b->num_blocks, b->max_blocks_per_seq,
                       b->scale, b->dtype, b->partition_tokens, b->workspace, b->workspace_bytes,
                       b->d_out, dev_err, stream);
  if (st != PA_OK) return st;

  // 4. download, behind the decode (on its own stream when pipelined); then
  // mark this set's device staging free for its next uploads
  if (piped) {
    if ((st = cuda_check(cudaEventRecord(compute_done, stream), "record decode")) != PA_OK) return st;
    if ((st = cuda_check(cudaStreamWaitEvent(ds, compute_done, 0), "order download")) != PA_OK) return st;
  }
  if ((st = cuda_check(cudaMemcpyAsync(out_host, b->d_out, q_bytes(b, n), cudaMemcpyDeviceToHost, ds), "download out")) != PA_OK) return st;
  if (piped && (st = cuda_check(cudaEventRecord(download_done, ds), "record download")) != PA_OK) return st;
  if (synchronize && (st = cuda_check(cudaStreamSynchronize(ds), "synchronize")) != PA_OK) return st;
  return ok();
}

pa_status_t pa_step_pipeline_create(pa_step_buffers_t* b, void* copy_stream, void* download_stream) {
  if (b == nullptr || copy_stream == nullptr || download_stream == nullptr)
    return fail(PA_ERR_INVALID_ARG, "buffers, copy_stream or download_stream is NULL");
  cudaEvent_t ev[3] = {nullptr, nullptr, nullptr};
  for (int i = 0; i < 3; ++i) {
    pa_status_t st = cuda_check(cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming), "create event");
    if (st != PA_OK) {
      for (int k = 0; k < i; ++k) cudaEventDestroy(ev[k]);
      return st;
    }
  }
  b->upload_done = ev[0];
  b->compute_done = ev[1];
  b->download_done = ev[2];
  b->copy_stream = copy_stream;
  b->download_stream = download_stream;
  return ok();
}

pa_status_t pa_step_pipeline_destroy(pa_step_buffers_t* b) {
  if (b == nullptr) return fail(PA_ERR_INVALID_ARG, "buffers is NULL");
  if (b->upload_done) cudaEventDestroy(static_cast<cudaEvent_t>(b->upload_done));
  if (b->compute_done) cudaEventDestroy(static_cast<cudaEvent_t>(b->compute_done));
  if (b->download_done) cudaEventDestroy(static_cast<cudaEvent_t>(b->download_done));
  b->upload_done = b->compute_done = b->download_done = nullptr;
  b->copy_stream = b->download_stream = nullptr;
  return ok();
}

}  // extern "C"
