// Host launcher of the tensor-core causal attention (kernel in attention_tc.cuh).
#include <math.h>

#include "attention_tc.cuh"
#include "internal.h"

namespace gpt {

int launch_attention_bf16(const AttnLayout& L, int B, int nh, int T, int32_t* status, cudaStream_t s) {
    if (B == 0 || nh == 0 || T == 0) return GPT_OK;
    // 4-D maps with non-decreasing strides: {hs, head, t, b} when heads are interleaved inside a
    // position (the fused c_attn output), {hs, t, head, b} when each head is a contiguous [T, hs]
    // block (the standalone layout).
    const bool head_inner = L.sh <= L.st;
    CUtensorMap tq, tk, tv;
    uint64_t dims[4], strides[3];
    const uint32_t box_head_inner[4] = {attn::HS, 1, attn::BQ, 1};
    const uint32_t box_t_inner[4] = {attn::HS, attn::BQ, 1, 1};
    dims[0] = attn::HS;
    if (head_inner) {
        dims[1] = nh; dims[2] = T; dims[3] = B;
        strides[0] = L.sh * 2; strides[1] = L.st * 2; strides[2] = L.sb * 2;
    } else {
        dims[1] = T; dims[2] = nh; dims[3] = B;
        strides[0] = L.st * 2; strides[1] = L.sh * 2; strides[2] = L.sb * 2;
    }
    const uint32_t* box = head_inner ? box_head_inner : box_t_inner;
    int rc = make_tmap_bf16_4d(&tq, L.q, dims, strides, box);
    if (!rc) rc = make_tmap_bf16_4d(&tk, L.k, dims, strides, box);
    if (!rc) rc = make_tmap_bf16_4d(&tv, L.v, dims, strides, box);
    if (rc) return rc;

    attn::Params p{};
    p.B = B;
    p.nh = nh;
    p.T = T;
    p.head_inner = head_inner ? 1 : 0;
    p.y = L.y;
    p.y_sb = L.y_sb;
    p.y_sh = L.y_sh;
    p.y_st = L.y_st;
    p.scale_log2 = static_cast<float>(1.4426950408889634 / sqrt(static_cast<double>(attn::HS)));
    p.status = status;
    p.lse = L.lse;

    static size_t opted[kMaxDevices] = {};
    rc = opt_in_smem(reinterpret_cast<const void*>(attn::attention_fwd_tc), attn::SMEM_BYTES, opted);
    if (rc) return rc;
    const long long n_qt = (T + attn::BQ - 1) / attn::BQ;
    const long long blocks = n_qt * B * nh;
    if (blocks > 0x7fffffffLL) return GPT_ERR_UNSUPPORTED;
    return launch_overlapped(attn::attention_fwd_tc, dim3(static_cast<unsigned>(blocks)), dim3(attn::THREADS),
                             attn::SMEM_BYTES, s, tq, tk, tv, p);
}

// Pipeline-wait limit of this file's kernels on the current device (0: the default).
GPT_DEFINE_WAIT_LIMIT_SETTER(set_wait_limit_attention)

}  // namespace gpt
