// sampler_noalloc.cu -- dg_sample without a caller-provided workspace.
//
// Some callers cannot allocate device memory at all: a serving process that has handed every free
// byte of HBM to its own pool allocator, a real-time loop where the synchronisation an allocation
// may cause is not allowed, or a plain C component that receives logits from elsewhere and owns no
// CUDA allocator.  For them dg_sample_noalloc runs the same two sampler kernels as dg_sample with
// their per-(row, vocabulary chunk) partial results kept in a static device array of this file.
//
// The array (kNoAllocSlots records of 8 floats = 1 MiB) is part of the loaded library: every GPU
// that loads libdg.so holds its own copy until the process exits.  Host code cannot use the
// array's name as a device address (on the host it names a host-side stand-in), so the first call
// on each device looks the device address up with cudaGetSymbolAddress, with that device current,
// and caches it for the life of the process; that first call should therefore happen before any
// stream capture, and a cudaDeviceReset after it is not supported (the reset unloads the module, so
// the cached address would point at freed memory).  All calls on
// a device share the one array and it keeps the last call's contents; nothing in it has to start
// at zero (every record is written by the partial kernel before the finalize kernel reads it).
// Calls that overlap on the GPU (different streams, or different threads without ordering) race
// on the array and must not be issued.
#include <cuda_runtime.h>
#include <stdio.h>

#include <mutex>

#include "dg.h"
#include "dg_kernels.h"

#define DG_API extern "C" __attribute__((visibility("default")))

namespace {

constexpr int kNoAllocSlots = 32768;   // (row, vocabulary chunk) records
constexpr int kMaxDevices = 64;

static __device__ __align__(256) float g_sample_partials[kNoAllocSlots * 8];

std::mutex g_mu;
float* g_addr[kMaxDevices] = {};

// Device address of g_sample_partials on the current device (looked up once per device).
cudaError_t scratch_address(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_sample_partials);
    if (e != cudaSuccess) return e;
    g_addr[dev] = static_cast<float*>(p);
  }
  *out = g_addr[dev];
  return cudaSuccess;
}

}  // namespace

DG_API size_t dg_sample_noalloc_max_rows(int vocab) {
  if (vocab <= 0 || vocab % 1024) return 0;   // vocabularies the sampler rejects
  return (size_t)kNoAllocSlots / (size_t)dg::sampler_chunks(vocab);
}

DG_API dg_status dg_sample_noalloc(const float* d_logits, int n_seq, int vocab, const dg_sampler_params* p, int step,
                                   const int32_t* d_seq_P, int32_t* d_ids, uint8_t* d_commit, float* d_entropy,
                                   int32_t* d_stop, void* stream) {
  if (!d_logits || !p || !d_ids || !d_commit || !d_entropy || !d_stop)
    return dg::record_error(DG_ERR_INVALID_ARG, "dg_sample_noalloc: null argument");
  if (n_seq <= 0 || vocab <= 0 || vocab % 1024)
    return dg::record_error(DG_ERR_INVALID_ARG, "dg_sample_noalloc: bad n_seq / vocab");
  if (step < 0) return dg::record_error(DG_ERR_INVALID_ARG, "dg_sample_noalloc: bad step");
  const dg_status ps = dg::check_sampler_params(p, step, "dg_sample_noalloc: ");
  if (ps != DG_OK) return ps;
  const int chunks = dg::sampler_chunks(vocab);
  // compare in size_t before forming n_seq * 256 (no int overflow for any n_seq)
  if ((size_t)n_seq * 256u * (size_t)chunks > (size_t)kNoAllocSlots) {
    char msg[192];
    snprintf(msg, sizeof msg,
             "dg_sample_noalloc: %d canvases x 256 rows x %d vocabulary chunks exceed the static scratch of %d records",
             n_seq, chunks, kNoAllocSlots);
    return dg::record_error(DG_ERR_CAPACITY, msg);
  }
  float* scratch = nullptr;
  const cudaError_t e = scratch_address(&scratch);
  if (e != cudaSuccess) {
    char msg[160];
    snprintf(msg, sizeof msg, "dg_sample_noalloc: cudaGetSymbolAddress of the scratch failed: %s", cudaGetErrorString(e));
    return dg::record_error(DG_ERR_CUDA, msg);
  }
  dg::SamplerArgs a{};
  a.logits = d_logits;
  a.n_seq = n_seq;
  a.canvas = 256;
  a.vocab = vocab;
  a.n_chunks = chunks;
  a.seq_P = d_seq_P;
  a.ids_in = d_ids;
  a.commit_in = d_commit;
  a.ids_out = d_ids;
  a.commit_out = d_commit;
  a.entropy = d_entropy;
  a.stop = d_stop;
  a.partial = scratch;
  a.inv_temp = 1.0f / dg_temperature(p, step);
  a.seed = p->seed;
  a.step = step;
  a.max_steps = p->max_steps;
  a.fixed_steps = p->fixed_steps;
  a.entropy_bound = p->entropy_bound;
  a.stop_mean_entropy = p->stop_mean_entropy;
  a.rerand_entropy = p->rerand_entropy;
  a.commit_rule = p->commit_rule;
  const cudaError_t le = dg::sampler_run(a, static_cast<cudaStream_t>(stream));
  if (le != cudaSuccess) {
    char msg[160];
    snprintf(msg, sizeof msg, "dg_sample_noalloc: launch failed: %s", cudaGetErrorString(le));
    return dg::record_error(DG_ERR_CUDA, msg);
  }
  return DG_OK;
}
