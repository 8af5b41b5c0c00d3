// LM head + fused argmax for callers that cannot allocate device memory.
//
// Some callers run where cudaMalloc is off limits: code inside a CUDA-graph
// capture, an allocator-free inference runtime that hands out only the tensors
// it owns, or a plug-in host that forbids allocation after start-up.  For them
// this entry point takes its scratch space (the split-bf16 copy of the
// normalised hidden rows and the per-vocabulary-tile top-2 partials) from one
// fixed array in device global memory that the library defines at file scope.
// Every GPU that loads the library holds that array until the process exits.
//
// The computation is the one the verification step ends with: RMSNorm of each
// hidden row with the final norm weights, the LM-head product, and per row the
// best logit, its vocabulary index (lowest index on ties) and the runner-up.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstring>
#include <mutex>

#include "../../include/spec.h"
#include "common.cuh"
#include "kernels.h"

namespace spec {
namespace {

constexpr int kNoallocMaxRows = 64;      // tokens per call (one 64-token GEMM tile)
constexpr int kNoallocMaxHidden = 8192;  // d
constexpr int kNoallocMaxVocab = 262144; // V
constexpr size_t kSplitBytes = (size_t)2 * kNoallocMaxRows * kNoallocMaxHidden * 2;  // hi + lo rows, bf16
constexpr size_t kTop2Bytes = (size_t)(kNoallocMaxVocab / 128) * kNoallocMaxRows * 12;  // one Top2 per tile x row
constexpr size_t kSsBytes = (size_t)kNoallocMaxRows * 4;
constexpr size_t kErrBytes = 256;  // the call's device error word (4 bytes used)
constexpr size_t kScratchBytes = kSplitBytes + kTop2Bytes + kSsBytes + kErrBytes;  // 3.5 MiB + 512 B

// The scratch.  In host code this name is only a stand-in for the device
// array: its device address comes from cudaGetSymbolAddress, once per device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

// per row: sum of squares of x, and x * w as split bf16 (the GEMM epilogue
// applies rsqrt(mean + eps))
__global__ void __launch_bounds__(256) noalloc_prep_kernel(const float* __restrict__ hidden,
                                                           const __nv_bfloat16* __restrict__ w, int d,
                                                           __nv_bfloat16* __restrict__ split, float* __restrict__ ss) {
  __shared__ float red[8];
  const int r = blockIdx.x;
  const float* x = hidden + (size_t)r * d;
  float s = 0.f;
  for (int k = threadIdx.x; k < d; k += blockDim.x) {
    const float v = x[k];
    s += v * v;
    split_store(split, r, d, k, v * __bfloat162float(w[k]));
  }
  s = warp_sum(s);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) t += red[i];
    ss[r] = t;
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// resolved once, in setup_device under g_setup_mu, before any encode() call
EncodeTiledFn g_encode = nullptr;

bool encode(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  const EncodeTiledFn fn = g_encode;
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// once-per-device set-up: the scratch's device address and kernel attributes
constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
unsigned char* g_scratch_ptr[kMaxDevices] = {};
int g_sm_count[kMaxDevices] = {};

int setup_device(int dev, unsigned char** scratch, int* sms) {
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (!g_encode) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return SPEC_ERR_CUDA;
    g_encode = reinterpret_cast<EncodeTiledFn>(p);
  }
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) {
      return SPEC_ERR_CUDA;
    }
    cudaDeviceProp prop;
    e = cudaGetDeviceProperties(&prop, dev);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(gemm_tc_function(64), cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)gemm_tc_smem_bytes(64));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(gemm_tc_function(64), cudaFuncAttributePreferredSharedMemoryCarveout,
                               (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) {
      return SPEC_ERR_CUDA;
    }
    g_sm_count[dev] = prop.multiProcessorCount;
    g_scratch_ptr[dev] = static_cast<unsigned char*>(p);
  }
  *scratch = g_scratch_ptr[dev];
  *sms = g_sm_count[dev];
  return SPEC_OK;
}

}  // namespace
}  // namespace spec

using namespace spec;

extern "C" {

int spec_lm_head_argmax_noalloc(const float* hidden, const void* final_norm, const void* lm_head, int M, int d, int V,
                                float eps, int32_t* argmax, float* top1, float* top2, void* cuda_stream) {
  if (!hidden || !final_norm || !lm_head || !argmax || !top1 || !top2) {
    return SPEC_ERR_ARG;
  }
  if (M < 1 || M > kNoallocMaxRows || d < 128 || d % 128 || d > kNoallocMaxHidden || V < 2 || V > kNoallocMaxVocab) {
    return SPEC_ERR_CAPACITY;
  }
  if (!(eps > 0.f) || (reinterpret_cast<uintptr_t>(lm_head) & 15u)) {
    return SPEC_ERR_ARG;
  }
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    return SPEC_ERR_CUDA;
  }
  unsigned char* scratch = nullptr;
  int sms = 0;
  int rc = setup_device(dev, &scratch, &sms);
  if (rc) return rc;
  __nv_bfloat16* split = reinterpret_cast<__nv_bfloat16*>(scratch);
  Top2* top_part = reinterpret_cast<Top2*>(scratch + kSplitBytes);
  float* ss = reinterpret_cast<float*>(scratch + kSplitBytes + kTop2Bytes);
  uint32_t* err = reinterpret_cast<uint32_t*>(scratch + kSplitBytes + kTop2Bytes + kSsBytes);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(cuda_stream);

  CUtensorMap map_lm, map_x;
  if (!encode(&map_lm, lm_head, (uint64_t)V, (uint64_t)d, 128) ||
      !encode(&map_x, split, 2 * (uint64_t)kNoallocMaxRows, (uint64_t)d, 128)) {
    return SPEC_ERR_CUDA;
  }
  // the error word starts every call at zero (a memset needs no allocation)
  e = cudaMemsetAsync(err, 0, sizeof(uint32_t), st);
  if (e != cudaSuccess) {
    return SPEC_ERR_CUDA;
  }
  noalloc_prep_kernel<<<M, 256, 0, st>>>(hidden, reinterpret_cast<const __nv_bfloat16*>(final_norm), d, split, ss);
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    return SPEC_ERR_CUDA;
  }
  GemmTcLaunch g{};
  g.bn = 64;
  g.epi = GEMM_EPI_ARGMAX;
  g.mA0 = g.mA1 = g.mA2 = &map_lm;
  g.mB = &map_x;
  g.args.n_out = V;
  g.args.K = d;
  g.args.M = M;
  g.args.tiles_o = (V + 127) / 128;
  g.args.tiles_t = 1;
  g.args.splits = 1;
  g.args.kb_per_split = d / 64;
  g.args.seg_rows[0] = V;
  g.args.ss_in = ss;
  g.args.n_ss = 1;
  g.args.ss_ld = kNoallocMaxRows;
  g.args.norm_d = d;
  g.args.eps = eps;
  g.args.top_part = top_part;
  g.args.top_ld = kNoallocMaxRows;
  g.args.err = err;
  g.grid = g.args.tiles_o < 2 * sms ? g.args.tiles_o : 2 * sms;
  e = gemm_tc_launch(g, st, false);
  if (e == cudaSuccess) e = launch_top2_reduce(M, g.args.tiles_o, top_part, kNoallocMaxRows, argmax, top1, top2, st, false,
                                                  err);
  if (e != cudaSuccess) {
    return SPEC_ERR_CUDA;
  }
  return SPEC_OK;
}

}  // extern "C"
