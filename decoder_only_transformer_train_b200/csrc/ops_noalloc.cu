// Attention backward whose only scratch, the per-row sums D = rowsum(dO * O), lives in a
// fixed array compiled into the library, so that the call allocates no device memory.
//
// Who needs it: a caller that holds only the operand buffers and cannot allocate, e.g. a
// C program with no allocator of its own, or one whose device memory is reserved up front
// by a caching allocator (a fresh cudaMalloc would fail or fragment that pool) and that
// cannot afford the device-wide synchronisation a cudaFree implies.  The caller-scratch
// entry point gpt2op_attention_bwd remains the general one; this one only changes where D
// lives and caps its size.
//
// What is shared: one array per device for the whole process.  Two calls whose executions
// overlap on the same device (different streams, or host threads launching concurrently)
// race on it.  Calls on one stream, or ordered by events, are safe.
//
// What must start at zero: nothing.  The first kernel of the call writes all B*H*T row sums
// before the kernels that read them run (same stream), and those only read rows < T.
#include <mutex>

#include "gpt2_b200.h"
#include "common.cuh"
#include "kernels.h"

namespace {

// Fixed scratch: GPT2OP_NOALLOC_ATTN_MAX_ROWS floats (1 MiB).  The kernels write and read D
// one float per (batch, head, query) row, so float alignment is all they need; the array is
// 256-byte aligned like cudaMalloc memory, so it meets anything the caller-scratch path may
// assume of its D buffer.
static __device__ __align__(256) float g_attn_rowsum_scratch[GPT2OP_NOALLOC_ATTN_MAX_ROWS];

constexpr int kMaxDevices = 64;
std::mutex g_addr_mutex;
float* g_addr[kMaxDevices] = {};

// Device address of the scratch on the current device, looked up once per device with
// cudaGetSymbolAddress (on the first call made on that device) and cached.
int scratch_address(float** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GPT2_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return GPT2_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_addr_mutex);
  if (g_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_attn_rowsum_scratch) != cudaSuccess || p == nullptr) return GPT2_ERR_CUDA;
    g_addr[dev] = static_cast<float*>(p);
  }
  *out = g_addr[dev];
  return GPT2_OK;
}

}  // namespace

extern "C" int gpt2op_attention_bwd_noalloc(void* stream, int precision, const void* qkv, const void* out,
                                            const void* dout, const float* lse, void* dqkv, int B, int T, int H,
                                            int head_dim) {
  if (!qkv || !out || !dout || !lse || !dqkv) return GPT2_ERR_ARG;
  if (precision != GPT2_FP32 && precision != GPT2_BF16) return GPT2_ERR_ARG;
  // Size checks come before any CUDA call, so an oversized request touches nothing.
  if (B <= 0 || T <= 0 || H <= 0 || head_dim <= 0) return GPT2_ERR_SHAPE;
  if ((long long)B * H * T > (long long)GPT2OP_NOALLOC_ATTN_MAX_ROWS) return GPT2_ERR_SHAPE;
  float* Dbuf = nullptr;
  const int rc = scratch_address(&Dbuf);
  if (rc != GPT2_OK) return rc;
  const int lrc = launch_attn_bwd(reinterpret_cast<cudaStream_t>(stream), precision == GPT2_BF16, qkv, out, dout,
                                  lse, Dbuf, dqkv, B, T, H, head_dim);
  return lrc == 0 ? GPT2_OK : (lrc == -4 ? GPT2_ERR_SHAPE : (lrc == -1 ? GPT2_ERR_ARG : GPT2_ERR_CUDA));
}
