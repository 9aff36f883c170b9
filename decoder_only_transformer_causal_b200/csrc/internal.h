// Host-side launchers shared by the C ABI (gpt_abi.cu) and the kernel files.  Every
// launcher validates nothing beyond what its kernel needs; argument checking against the
// public contract happens in gpt_abi.cu.  All return a GPT_* status.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/gpt.h"

namespace gpt {

typedef __nv_bfloat16 bf16;

int num_sms();
int cuda_status(cudaError_t e);

// Opts a kernel in for `bytes` of dynamic shared memory on the current device.  `opted` is a
// per-kernel table (a function-local static of the caller) of the size each device is opted in
// for; the attribute is set the first time a device needs a size, or a larger one.
constexpr int kMaxDevices = 64;
int opt_in_smem(const void* kern, size_t bytes, size_t (&opted)[kMaxDevices]);

// Launches `kern` so that it may overlap the tail of the previous kernel in the stream
// (programmatic stream serialisation); every kernel launched this way calls griddep_wait()
// before touching memory its predecessor uses.
template <typename... KArgs, typename... Args>
int launch_overlapped(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                      Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cuda_status(cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...));
}

// The same in clusters of `cluster_x` CTAs along x; grid.x must be a multiple of it.
template <typename... KArgs, typename... Args>
int launch_overlapped_cluster(void (*kern)(KArgs...), unsigned cluster_x, dim3 grid, dim3 block, size_t smem,
                              cudaStream_t s, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster_x;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cuda_status(cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...));
}

// Clusters of two CTAs (the 2-SM MMA's pairs); grid.x must be even.
template <typename... KArgs, typename... Args>
int launch_overlapped_pairs(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                            Args&&... args) {
    return launch_overlapped_cluster(kern, 2u, grid, block, smem, s, static_cast<Args&&>(args)...);
}

// ---- TMA descriptors (cuTensorMapEncodeTiled through the runtime's driver entry point)
int make_tmap_bf16_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                      uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer);
// 2-D map with 64-byte swizzle for epilogue staging tiles (box rows of 64 bytes); fp32 or bf16.
int make_tmap_2d_sw64(CUtensorMap* m, const void* base, bool fp32, uint64_t inner, uint64_t outer,
                      uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer);
int make_tmap_bf16_4d(CUtensorMap* m, const void* base, const uint64_t dims[4],
                      const uint64_t strides_bytes[3], const uint32_t box[4]);

// ---- row-wise kernels (rowwise.cu)
int launch_embed(const void* wte, const void* wpe, const int64_t* idx, float* x, int B, int T,
                 int C, int V, int dtype, int32_t* status, cudaStream_t s);
// xcopy (optional, 16-byte aligned): also writes the input rows there unchanged.
int launch_layernorm(const float* x, const void* w, const void* b, void* out, int rows, int C,
                     int dtype, cudaStream_t s, float* xcopy = nullptr);
// bf16 path: combine the lm_head epilogue's partials into per-row losses.
int launch_ce_rows_from_parts(const float2* part, int n_part, const float* tlogit,
                              const int64_t* targets, int rows, int V, float* row_loss,
                              int32_t* status, cudaStream_t s,
                              float* row_lse = nullptr);
// fp32 path: per-row losses straight from fp32 logits.
int launch_ce_rows_from_logits(const float* logits, const int64_t* targets, int rows, int V,
                               float* row_loss, int32_t* status, cudaStream_t s);
// Fixed-order sum of the counted rows' losses -> loss, {sum, count}.
int launch_loss_finalize(const float* row_loss, const int64_t* targets, int rows, int V,
                         float* loss, double* sum_count, cudaStream_t s);

// ---- tensor-core GEMM (gemm_tc.cu)
struct CeArgs {
    const int64_t* targets;
    float2* part;
    float* tlogit;
    int n_part;
};
int gemm_ce_parts(int N);  // partial slots per row of the lm_head epilogue
// launch_gemm_bf16 epilogue beyond GPT_EPI_*: out bf16 [2M, ldo] = {gelu'(acc + b); gelu(acc + b)},
// M % 32 == 0.
constexpr int GEMM_EPI_GELU2 = 6;
int launch_gemm_bf16(const bf16* A, long long lda, const bf16* W, long long ldw, const bf16* bias,
                     void* out, long long ldo, int M, int N, int K, int epilogue, int gelu,
                     const CeArgs* ce, int32_t* status, cudaStream_t s);

// out[M, N] (fp32, row stride ldo) += A B^T.  A: [M, K] (a_mn false) or stored as [K, M] (a_mn);
// W: [N, K] (b_mn false) or stored as [K, N] (b_mn); row strides lda / ldw in elements.  a_mn
// requires b_mn.  split_ws (optional, 16-byte aligned, gemm_acc_split_bytes(M, N, K) bytes): with
// a_mn, a product whose M x N tiles would leave SMs idle is split along K into partial products
// that a second pass adds to out in a fixed order (results independent of scheduling).
int launch_gemm_bf16_acc(const bf16* A, long long lda, bool a_mn, const bf16* W, long long ldw, bool b_mn, float* out,
                         long long ldo, int M, int N, int K, int32_t* status, cudaStream_t s,
                         float* split_ws = nullptr);
size_t gemm_acc_split_bytes(int M, int N, int K);
// Products of the backward with W stored [K, N] (b_mn, required):
//   GEMM_BWD_ACC_F32     out fp32 += A B^T (a_mn allowed; split-K as launch_gemm_bf16_acc)
//   GEMM_BWD_STORE_F32   out fp32  = A B^T
//   GEMM_BWD_STORE_BF16  out bf16  = A B^T
//   GEMM_BWD_DGELU_BF16  out bf16  = (A B^T) * aux, aux bf16 [M, ld_aux] the stored GELU derivative;
//                        with colsum, also its column sums per 32-row band into colsum
//                        [ceil(M / 32), N] (launch_colsum_bands finishes the bias gradient)
enum { GEMM_BWD_ACC_F32 = 0, GEMM_BWD_STORE_F32 = 1, GEMM_BWD_STORE_BF16 = 2, GEMM_BWD_DGELU_BF16 = 3 };
int launch_gemm_bf16_bwd(const bf16* A, long long lda, bool a_mn, const bf16* W, long long ldw, bool b_mn, void* out,
                         long long ldo, int M, int N, int K, int mode, const bf16* aux, long long ld_aux, int gelu,
                         int32_t* status, cudaStream_t s, float* split_ws = nullptr, float* colsum = nullptr);

// ---- tensor-core attention (attention_tc.cu); strides in elements
struct AttnLayout {
    const bf16 *q, *k, *v;
    long long sb, sh, st;  // strides of q/k/v for batch, head, position (hs contiguous)
    bf16* y;
    long long y_sb, y_sh, y_st;
    float* lse = nullptr;  // optional [B, nh, T]: log2 sum_j 2^(s_ij * scale_log2), for the backward
};
int launch_attention_bf16(const AttnLayout& L, int B, int nh, int T, int32_t* status, cudaStream_t s);

// Limit after which a pipeline wait of the tensor-core kernels gives up, on the current device,
// one setter per file holding such kernels (ns 0: the default 1 s), and the forced time-out of
// the testing aid (common.cuh, g_force_timeout).
int set_wait_limit_attention(unsigned long long ns, int force);
int set_wait_limit_gemm(unsigned long long ns, int force);
int set_wait_limit_attention_bwd(unsigned long long ns, int force);
int set_wait_limit_head(unsigned long long ns, int force);
int set_wait_limit_decode(unsigned long long ns, int force);

// ---- one decode step as a single cooperative kernel (decode_persistent.cu): bf16, B <= 16,
// C % 128 == 0 and C <= 1024, head size % 8 == 0 and <= 64, V % 8 == 0, and a shared-memory plan
// that fits.  bar: a word zeroed per launch (set here).
bool decode_persistent_supported(int dtype, int B, int C, int hs, int V, int has_bias);
int launch_decode_persistent(const void* wte, const void* wpe, const void* layer0, long long layer_bytes,
                             const long long (&off)[12], int has_bias, const void* lnf_w, const void* lnf_b,
                             const int64_t* tok, long long ld_tok, void* kv, long long kv_layer_elems, float* logits,
                             long long ldl, int* pos, float* x, void* q, void* y, void* h, float* part,
                             int* counter, int n_split_max, unsigned* bar, int32_t* status, int B, int C, int nh,
                             int V, int L, int block_size, int gelu_tanh, cudaStream_t s);

// ---- the inference branch's head (head_last.cu): logits[b, :] = LayerNorm(x_b; lnw, lnb) wte^T
// for B rows x + b * ldx (fp32, 16-byte aligned rows); logits bf16 at out + b * ldo.  C % 8 == 0
// and C <= 2048 (head_last_tc_supported).
bool head_last_tc_supported(int C);
int launch_head_last_bf16(const float* x, long long ldx, const bf16* lnw, const bf16* lnb, const bf16* wte, int B,
                          int C, int V, bf16* out, long long ldo, int32_t* status, cudaStream_t s);

// ---- fp32 SIMT path (simt_f32.cu)
int launch_linear_f32(const float* A, long long lda, const float* W, const float* bias, float* out,
                      long long ldo, int M, int N, int K, int epilogue, int gelu, cudaStream_t s);
struct AttnLayoutF32 {
    const float *q, *k, *v;
    long long sb, sh, st;
    float* y;
    long long y_sb, y_sh, y_st;
    float* lse = nullptr;  // optional [B, nh, T], as in AttnLayout
};
int launch_attention_f32(const AttnLayoutF32& L, int B, int nh, int T, int hs, cudaStream_t s);

// ---- incremental decoding and sampling (decode.cu); E = bf16 or fp32 by dtype
// x[b, :] = wte[tok[b * ld_tok]] + wpe[*pos] (fp32 x [B, C]).
int launch_embed_pos(const void* wte, const void* wpe, const int64_t* tok, long long ld_tok, const int* pos, float* x,
                     int B, int C, int V, int block_size, int dtype, int32_t* status, cudaStream_t s);
// Matrix-vector products of B rows against W [N, K]; epi 1 gelu -> E, 2 fp32 +=, 3 fp32
// store, 4 qkv split (q -> out, k/v -> kv[b, *pos]), 5 store E.  ln: the input is the fp32
// residual stream and LayerNorm(ln_w, ln_b) is applied to it first.  bump_pos: advance *pos by
// one.  gemv_smem_bytes: the dynamic shared memory a launch with `B` rows needs (the library's
// limit is 227 KB per CTA).
int launch_gemv(int epi, bool ln, int dtype, const void* x, long long ldx, const void* ln_w, const void* ln_b,
                const void* W, const void* bias, void* out, long long ldo, int B, int N, int K, int gelu_tanh,
                void* kv, int* pos, int C, int block_size, int bump_pos, cudaStream_t s);
size_t gemv_smem_bytes(int B, int K, int dtype, bool ln);
constexpr int kGemvEpiStore = 5;
size_t decode_attn_part_floats(int B, int nh, int hs, int block_size);
// counter: B * nh ints, zero on entry and on return.
int launch_decode_attention(int dtype, const void* q, const void* kv, const int* pos, float* part, int* counter,
                            void* y, int B, int nh, int hs, int block_size, cudaStream_t s);
int launch_kv_store(const void* qkv, void* kv, int B, int T, int C, int elem_bytes, int block_size, cudaStream_t s);
int launch_copy_tokens(const int64_t* src, long long ld_src, int64_t* dst, long long ld_dst, int B, int T,
                       cudaStream_t s);
// *pos = value and counter[0, n_counter) = 0.
int launch_decode_reset(int* pos, int value, int* counter, int n_counter, cudaStream_t s);
int sample_max_vocab();  // largest V the sampling kernel takes (the row sits in shared memory)
int launch_sample(const float* logits, long long ld_logits, int B, int V, float temperature, int top_k,
                  const float* u, int64_t* out, long long ld_out, cudaStream_t s);

// ---- optimizer step (optim.cu)
constexpr int kOptMaxTensors = 1024;
// The packed tensors in element units: tensor i spans [off[i], off[i] + numel[i]) of the flat
// fp32 arrays, is cut into chunks starting at chunk index chunk0[i] (chunk0[n] = total), and
// takes weight decay iff decay[i].
struct OptTable {
    int n;
    long long off[kOptMaxTensors];
    long long numel[kOptMaxTensors];
    long long chunk0[kOptMaxTensors + 1];
    unsigned char decay[kOptMaxTensors];
};
long long opt_chunk_elems();
size_t adamw_workspace_bytes();
int launch_adamw(const OptTable& tab, int dtype, float* params, const float* grads, float* m, float* v, void* copy,
                 float lr, float beta1, float beta2, float eps, float weight_decay, int step, float max_norm,
                 float* norm_out, void* ws, cudaStream_t s);

// ---- backward kernels of the non-matmul pieces (backward.cu)
// row_lse (optional): each row's logsumexp from the forward; the gradient then takes one pass.
int launch_ce_backward(const void* logits, int dtype, const int64_t* targets, const double* sum_count, void* dlogits,
                       int rows, int V, int32_t* status, cudaStream_t s, float scale = 1.f,
                       const float* row_lse = nullptr);
int layernorm_backward_parts(int rows, int C);  // part: [parts, 2C] floats ([parts, 3C] with dsum)
// dx16 (optional): a bf16 copy of the dx rows as written (the next products' operand).
// dsum (optional, needs accumulate_wb): dsum[c] += sum over rows of dx[r, c] as written, the bias
// gradient of the projection that added into the residual stream at this LayerNorm's input.
int launch_layernorm_backward(const float* dy, const float* x, const void* w, int dtype, float* dx, int accumulate,
                              float* dw, float* db, int accumulate_wb, float* part, int rows, int C, cudaStream_t s,
                              bf16* dx16 = nullptr, float* dsum = nullptr);
int colsum_parts(int rows);              // part: [parts, C] floats
// out[c] (+)= sum over i < n_part of part[i * C + c], in order of i (the second stage of the
// per-band column sums a producer kernel leaves).
int launch_colsum_bands(const float* part, int n_part, int C, float* out, int accumulate, cudaStream_t s);
int launch_colsum(const void* y, int dtype, int rows, int C, float* out, int accumulate, float* part,
                  cudaStream_t s);
int launch_gelu_backward(const float* dh, const void* pre, int dtype, void* dpre, long long n, int tanh_form,
                         cudaStream_t s);
int embed_backward_max_rows();
int launch_embed_backward(const int64_t* idx, const float* dx, int B, int T, int C, int V, float* dwte, float* dwpe,
                          unsigned long long* sorted, int32_t* status, cudaStream_t s);

// ---- training-step helpers and the attention backward (train.cu)
template <typename E>
struct AttnBwdLayout {
    const E *q, *k, *v;             // forward inputs, strides sb, sh, st (hs contiguous)
    long long sb, sh, st;
    const E *o, *dout;              // forward output and its gradient, strides o_sb, o_sh, o_st
    long long o_sb, o_sh, o_st;
    E *dq, *dk, *dv;                // gradients, with the q / k / v strides
    const float* lse;               // [B, nh, T] from the forward
};
int launch_transpose(const void* in, int in_dtype, long long ld_in, void* out, int out_dtype, long long ld_out, int R,
                     int Cc, cudaStream_t s);
int launch_gelu_forward(const void* pre, void* h, long long n, int dtype, int tanh_form, cudaStream_t s);
int launch_gelu_deriv_inplace(void* pre, long long n, int dtype, int tanh_form, cudaStream_t s);
// scratch: attn_bwd_scratch_bytes(B, nh, T) bytes, 16-byte aligned (D and lse2 padded to a multiple
// of 128 rows per head).  Exactly one of Lb / Lf is non-null; hs 32 or 64.  status: optional device
// word that records GPT_ERR_TIMEOUT from the tensor-core kernels.
size_t attn_bwd_scratch_bytes(long long B, long long nh, long long T);
// Column sums of dq / dk / dv per 32-row band of each sequence, left by the tensor-core kernels:
// part [B * ceil(T / 32), ld] floats; head h's columns of q, k, v start at col_q, col_k, col_v +
// h * hs (finish with launch_colsum_bands).
struct AttnBwdColsum {
    float* part;
    long long ld;
    int col_q, col_k, col_v;
};
// cs (optional): *cs_done says whether the band sums were written (the tensor-core kernels ran).
int launch_attention_backward(const AttnBwdLayout<bf16>* Lb, const AttnBwdLayout<float>* Lf, int B, int nh, int T,
                              int hs, float* scratch, int32_t* status, cudaStream_t s,
                              const AttnBwdColsum* cs = nullptr, bool* cs_done = nullptr);
// bf16, head size 64: returns GPT_ERR_BAD_ALIGN (nothing launched) when an operand cannot be
// described by a TMA map.
int launch_attention_backward_tc(const AttnBwdLayout<bf16>& L, int B, int nh, int T, const float* D,
                                 const float* lse2, int32_t* status, cudaStream_t s,
                                 const AttnBwdColsum* cs = nullptr);

}  // namespace gpt
