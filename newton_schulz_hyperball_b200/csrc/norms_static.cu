// Frobenius norms without any caller-provided workspace.
//
// nshb_fro_norms needs a device workspace for its per-block partial sums.  Some callers
// cannot hand one over: code that runs where it may not call cudaMalloc -- for instance a
// framework hook that computes rho = ||W0|| or monitors weight radii while the framework's
// own caching allocator has reserved the device memory and forbids allocations behind its
// back -- and callers that have no allocator of their own (C tools linking only this
// library).  nshb_fro_norms_static runs the same two kernels (block partials, then a
// fixed-order per-matrix sum) with its scratch in a fixed, file-scope device array.
//
// The array (NSHB_STATIC_SCRATCH_BYTES) is part of the module image, so every GPU that
// loads this library holds it until the process exits.  Host code cannot use the array's
// name as a device address; the address is looked up once per device with
// cudaGetSymbolAddress, with that device current, on the first call made on the device.
// Every call shares the array: calls that overlap on the GPU (different streams, or
// different host threads on one device) race and must be serialised by the caller.
// The looked-up address is kept for the life of the process, so a device reset
// (cudaDeviceReset) after the first call on that device is not supported.  A non-finite
// norm shows only as a NaN or Inf in the output: there is no status word to read.
#include <cuda_runtime.h>

#include <cstring>
#include <mutex>

#include "../../include/nshb.h"
#include "nshb_internal.h"

namespace nshb {
namespace {

constexpr size_t kScratchBytes = NSHB_STATIC_SCRATCH_BYTES;
constexpr size_t kStatusBytes = 256;                                  // status word + counter
constexpr int kStaticMaxMats = 192;                                   // matrices per call
constexpr size_t kScalarsBytes = sizeof(MatScalars) * kStaticMaxMats; // per-matrix records
constexpr size_t kPartialsOff = kStatusBytes + ((kScalarsBytes + 255) / 256) * 256;
constexpr size_t kMaxBlocks = (kScratchBytes - kPartialsOff) / (3 * sizeof(double));
static_assert(kStaticMaxMats <= kMaxMats, "one launch of the norm kernels");

__device__ __align__(256) unsigned char g_norm_scratch[kScratchBytes];

std::mutex g_mu;
char *g_addr[64] = {nullptr};

// Device address of g_norm_scratch on the current device (looked up once per device).
nshb_status scratch_address(char **out) {
  int dev = 0;
  const cudaError_t de = cudaGetDevice(&dev);
  if (de != cudaSuccess) {
    record_cuda_error(de);
    return NSHB_ERR_CUDA;
  }
  if (dev < 0 || dev >= 64) return NSHB_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> g(g_mu);
  if (!g_addr[dev]) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_norm_scratch);
    if (e != cudaSuccess || !p) {
      record_cuda_error(e != cudaSuccess ? e : cudaErrorInvalidSymbol);
      return NSHB_ERR_CUDA;
    }
    g_addr[dev] = static_cast<char *>(p);
  }
  *out = g_addr[dev];
  return NSHB_OK;
}

}  // namespace
}  // namespace nshb

using namespace nshb;

extern "C" nshb_status nshb_fro_norms_static(const nshb_matrix *mats, int32_t n_mats, float *out,
                                             nshb_stream stream) {
  if (n_mats < 0) return NSHB_ERR_SHAPE;
  if (n_mats == 0) return NSHB_OK;
  if (!mats || !out) return NSHB_ERR_NULL;
  if ((uintptr_t)out % sizeof(float)) return NSHB_ERR_SHAPE;
  if (n_mats > kStaticMaxMats) return NSHB_ERR_WORKSPACE;
  ApplyParams ap;
  ApplyFinParams fp;
  std::memset(&ap, 0, sizeof(ap));
  std::memset(&fp, 0, sizeof(fp));
  size_t blocks = 0;
  for (int i = 0; i < n_mats; ++i) {
    const nshb_matrix &d = mats[i];
    const nshb_status ce = check_matrix(d, nullptr, false, /*w_only=*/true);
    if (ce != NSHB_OK) return ce;
    const bool wf32 = d.w_dtype == NSHB_F32;
    const size_t esz = wf32 ? 4 : 2;
    const bool vec = ((uintptr_t)d.W % 16 == 0) && ((d.ld * esz) % 16 == 0);
    MatDesc &md = ap.mats[i];
    md.W = d.W;
    md.m = (int)d.rows;
    md.n = (int)d.cols;
    md.ld = (int)d.ld;
    md.flags = (vec ? kVec : 0) | (wf32 ? kWF32 : 0);
    md.pr = (int)((d.rows + kBlk - 1) / kBlk * kBlk);
    md.pc = (int)((d.cols + kBlk - 1) / kBlk * kBlk);
    md.blk_begin = (int)blocks;
    md.rec_begin = (int)blocks;
    md.mat = i;
    fp.rec_begin[i] = (int)blocks;
    fp.blk_begin[i] = (int)blocks;
    fp.mat[i] = i;
    fp.m[i] = md.m;
    fp.n[i] = md.n;
    blocks += (size_t)(md.pr / kBlk) * (md.pc / kBlk);
    if (blocks > kMaxBlocks) return NSHB_ERR_WORKSPACE;  // beyond the fixed scratch
  }
  fp.blk_begin[n_mats] = (int)blocks;
  fp.rec_begin[n_mats] = (int)blocks;

  char *scratch = nullptr;
  nshb_status e = scratch_address(&scratch);
  if (e != NSHB_OK) return e;
  cudaStream_t st = (cudaStream_t)stream;
  uint32_t *status = reinterpret_cast<uint32_t *>(scratch);
  MatScalars *scal = reinterpret_cast<MatScalars *>(scratch + kStatusBytes);
  double *partials = reinterpret_cast<double *>(scratch + kPartialsOff);
  // The status word and the exact-pass counter start at zero; partials and records are
  // fully written by the kernels before they are read.
  cudaError_t ce = cudaMemsetAsync(status, 0, 2 * sizeof(uint32_t), st);
  if (ce != cudaSuccess) {
    record_cuda_error(ce);
    return NSHB_ERR_CUDA;
  }
  ap.ws = scratch;
  ap.partials = partials;
  ap.scal = scal;
  ap.status = status;
  ap.op = kOpNorms;
  ap.nmat = n_mats;
  ap.total_blocks = (int)blocks;
  fp.partials = partials;
  fp.scal = scal;
  fp.status = status;
  fp.norms_out = out;
  fp.op = kOpNorms;
  fp.stage = 0;
  fp.hb_eps = 1e-8f;
  fp.nmat = n_mats;
  ce = launch_reduce(ap, st);
  if (ce == cudaSuccess) ce = launch_apply_finalize(fp, st);
  if (ce != cudaSuccess) {
    record_cuda_error(ce);
    return NSHB_ERR_CUDA;
  }
  return NSHB_OK;
}
