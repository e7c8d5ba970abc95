// nc_attention_noalloc: the attention layer of nc_attention (RoPE + QK-norm,
// then windowed causal attention) for callers that cannot hand the library a
// workspace.  Its scratch (the RoPE tables and the normalised q and k) lives
// in one fixed-size array in device memory that the library owns.
#include <mutex>

#include "nc_internal.cuh"

namespace nc {
namespace {

constexpr size_t kScratchBytes = size_t(32) << 20;  // 32 MiB per device, held until the process exits

__device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDev = 64;
unsigned char* g_scratch_ptr[kMaxDev];
bool g_scratch_ready[kMaxDev];
std::mutex g_scratch_mu;

// Device address of this device's scratch array.  Host code cannot use the
// array's name as a device pointer (it names a host-side shadow), so the
// address is looked up once per device, with that device current.
bool scratch_on_current_device(unsigned char** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDev) {
    record_error("nc_attention_noalloc: cudaGetDevice", e != cudaSuccess ? e : cudaErrorInvalidDevice);
    return false;
  }
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_ready[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      record_error("nc_attention_noalloc: cudaGetSymbolAddress", e != cudaSuccess ? e : cudaErrorInvalidSymbol);
      return false;
    }
    g_scratch_ptr[dev] = static_cast<unsigned char*>(p);
    g_scratch_ready[dev] = true;
  }
  *out = g_scratch_ptr[dev];
  return true;
}

size_t align256(size_t b) { return (b + 255) & ~size_t(255); }

}  // namespace

// status word lives in nc_api.cu
bool status_word(int** out);

}  // namespace nc

using namespace nc;

extern "C" size_t nc_attention_noalloc_max_bytes(void) { return kScratchBytes; }

extern "C" int nc_attention_noalloc(const void* q, const void* k, const void* v, void* out, int B, int T, int H,
                                    int Hkv, int D, int window, float alpha, float softmax_scale,
                                    float rope_base, float eps, int dtype, void* stream) {
  reset_launch_count();
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr) return NC_ERR_ARG;
  if (dtype != NC_BF16 && dtype != NC_FP32) return NC_ERR_ARG;
  if (!(softmax_scale > 0.f) || !(eps >= 0.f)) return NC_ERR_ARG;
  if (B <= 0 || T <= 0 || H <= 0 || Hkv <= 0 || D != 128 || H % Hkv != 0) return NC_ERR_SHAPE;
  const uintptr_t mis = (reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                         reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(out)) & 15u;
  if (mis) return NC_ERR_ALIGN;
  // scratch layout: cos table | sin table | q-hat | k-hat
  const size_t esz = dtype == NC_BF16 ? 2 : 4;
  const size_t M = (size_t)B * T;
  const size_t tab = align256((size_t)T * (D / 2) * 4);
  const size_t qb = align256(M * H * D * esz);
  const size_t kb = align256(M * Hkv * D * esz);
  if (2 * tab + qb + kb > kScratchBytes) return NC_ERR_WORKSPACE;  // beyond the fixed maximum
  unsigned char* base = nullptr;
  if (!scratch_on_current_device(&base)) return NC_ERR_CUDA;
  int* status = nullptr;
  if (!status_word(&status)) return NC_ERR_CUDA;
  int sms = 0, dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) {
    record_error("nc_attention_noalloc: device query", e);
    return NC_ERR_CUDA;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* rc = reinterpret_cast<float*>(base);
  float* rs = reinterpret_cast<float*>(base + tab);
  void* qo = base + 2 * tab;
  void* ko = base + 2 * tab + qb;
  const int bf = dtype == NC_BF16;
  const int w = (window <= 0 || window >= T) ? T : window;
  // every byte of scratch a kernel reads is written earlier in this same call
  launch_rope_table(rc, rs, T, D, rope_base, st);
  launch_rope_qknorm_copy(q, k, qo, ko, B, T, H, Hkv, D, rc, rs, alpha, eps, bf, st);
  if (bf) {
    if (!launch_attn_tc((const bf16*)qo, (const bf16*)ko, (const bf16*)v, H * D, Hkv * D, Hkv * D, (bf16*)out,
                        H * D, B, T, H, Hkv, w, softmax_scale, status, sms, st)) {
      check_launch("nc_attention_noalloc");
      return NC_ERR_CUDA;
    }
  } else {
    launch_attn_simt(qo, ko, v, H * D, Hkv * D, Hkv * D, out, H * D, B, T, H, Hkv, w, softmax_scale, bf, st);
  }
  return check_launch("nc_attention_noalloc");
}
