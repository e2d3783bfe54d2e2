// Host launchers of the memory-bound kernels of the training step.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>
#include <functional>
#include "gemm.h"

// Device error code of the top-k sampling kernel, next to the codes of the training step
// (DEVERR_NONE .. DEVERR_INTERNAL = 4 in common.cuh).
constexpr int DEVERR_ROW = 5;   // a sampled row index outside the logits

struct AdamBlock {      // one block of the multi-tensor AdamW launch
  long long off;        // first element (flat parameter index)
  int n;                // elements in this block
  int decay;            // 1 if weight decay applies to this tensor
};

// act = float (fp32 mode) or bf16 (bf16 mode), chosen by `bf16`.
int launch_encoder_fwd(cudaStream_t st, const int* tok, const float* wte, const float* wpe, float* x, int N, int T,
                       int C, int V);
int launch_layernorm_fwd(cudaStream_t st, bool bf16, const float* x, const float* w, const float* b, void* y,
                         float* mean, float* rstd, int N, int C);
// dy: the gradient of the LayerNorm output, of the activation type (bf16 in bf16 mode, as the
// bf16 product that makes it returns it).  part: nblocks rows of 3C floats, each the column
// sums over this block's rows of [dy * xhat | dy | new dres] (the weight, bias and upstream
// Linear bias gradients), left for launch_colsum_batch.
int launch_layernorm_bwd(cudaStream_t st, bool bf16, const void* dy, const float* x, const float* mean,
                         const float* rstd, const float* w, float* dres, void* dres_act, bool accumulate,
                         float* part, int nblocks, int N, int C);
int layernorm_bwd_blocks(int num_sms);
int launch_colsum(cudaStream_t st, bool bf16, const void* x, long long ldx, int M, int N, float* part, int nchunks,
                  float* out);
int colsum_chunks(int M);
int launch_ce_finalize(cudaStream_t st, const CePartial* part, int n_tiles, const float* zt, const int* targets,
                       int N, int V, float* lse, float* loss_row, int* argmax);
int launch_ce_rowwise(cudaStream_t st, const float* logits, long long ld, const int* targets, int N, int Vp, int V,
                      float* lse, float* loss_row, int* argmax);
int launch_loss_reduce(cudaStream_t st, const float* loss_row, const int* targets, int N, float grad_scale,
                       float* loss_out, float* dz_scale_out, int* count_out);
int launch_ce_dz(cudaStream_t st, bool bf16, void* logits, long long ld, const float* lse, const int* targets,
                 const float* dz_scale, int N, int Vp);
// Positions one embedding backward may take (B*T).
constexpr int ENC_MAX_POSITIONS = 131072;
// sorted_keys: N uint64 (token << 32 | position, ascending); seg_keys: encoder_bwd_seg_words(N)
// uint32 of scratch; chunk_part: encoder_bwd_part_floats(N, C) floats.
int launch_encoder_bwd(cudaStream_t st, const int* tok, const float* dx0, float* dwte, float* dwpe, int B, int T,
                       int C, uint64_t* sorted_keys, uint32_t* seg_keys, float* chunk_part, int V);
size_t encoder_bwd_part_floats(int N, int C);
size_t encoder_bwd_seg_words(int N);
int launch_topk_sample(cudaStream_t st, bool is_bf16, const void* logits, long long ld, int n_rows, const int* rows,
                       const float* u, int n, int V, int k, int* out, int* out_topk);
int launch_global_norm(cudaStream_t st, const float* g, long long n, double* part, int nparts, float clip,
                       float* out2);
int launch_adamw(cudaStream_t st, float* p, const float* g, float* m, float* v, uint16_t* shadow,
                 const AdamBlock* blocks, int nblocks, const float* clip_scale, float lr, float b1, float b2,
                 float eps, float wd, float bc1, float bc2);
int launch_init_normal(cudaStream_t st, float* p, long long n, uint64_t state, double std);
int launch_fill(cudaStream_t st, float* p, long long n, float value);
int launch_cast_bf16(cudaStream_t st, const float* src, uint16_t* dst, long long n);
int launch_attn_fwd(cudaStream_t st, bool bf16, const void* qkv, void* out, float* lse, int B, int T, int H,
                    int hd);
// bias_part (may be null; the bf16 head-size-64 path only): column sums of dqkv per 32-row
// lane quarter of each 128-row tile, attn_bwd_bias_rows(B, T) rows of 3C floats, to be
// reduced by launch_colsum_batch into the c_attn bias gradient.
int launch_attn_bwd(cudaStream_t st, bool bf16, const void* qkv, const void* out, const void* dout,
                    const float* lse, float* Dbuf, void* dqkv, int B, int T, int H, int hd,
                    float* bias_part = nullptr);
int launch_attn_fwd_tc(cudaStream_t st, const void* qkv, void* out, float* lse, int B, int T, int H, int hd);
int launch_attn_bwd_tc(cudaStream_t st, const void* qkv, const void* dout, const float* lse, const float* Dbuf,
                       void* dqkv, int B, int T, int H, int hd, float* bias_part);
inline int attn_bwd_bias_rows(int B, int T) { return (T + 127) / 128 * B * 4; }
// One fixed-order column reduction: out[n] += sum over k < rows of part[k * ld + n], n < ncols.
struct ColsumJob {
  const float* part;
  float* out;
  int ld;
  int rows;
  int ncols;
};
// Runs every job, up to 100 per launch; each output element gets one add of its sum, whose
// order of terms is fixed.  Jobs must not write overlapping outputs; their column counts and
// row strides must be multiples of 4 floats and their pointers 16-byte aligned (-1 if not).
int launch_colsum_batch(cudaStream_t st, const ColsumJob* jobs, int njobs);
int read_and_clear_device_error(int* code);
// Host-side values computed once per (key, device) under a lock: a process may drive several
// GPUs, from several threads, and a kernel attribute set on one device is unset on the others.
// compute() runs with the key's device current; negative results are returned, not cached.
int per_device_once(const void* key, const std::function<int()>& compute);
int current_device_sms();   // SM count of the current device (148 if the query fails)
// Raises `func`'s dynamic shared-memory limit to `bytes` on the current device, once per
// device (0, or -3 if the runtime refuses).
int set_dynamic_smem_once(const void* func, int bytes);
// Host-side count of the kernels launched by this library (for benchmark reporting).
void note_kernel_launches(int n);
long long kernel_launch_count();
