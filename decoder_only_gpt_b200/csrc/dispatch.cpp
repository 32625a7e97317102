// Kernel selection by storage type: bf16 contractions run on the tcgen05
// kernels (GEMM, attention forward), the fp32 configuration on CUDA cores.
#include "gpt_internal.h"

namespace gpt {

int launch_gemm_tc(const GemmArgs& g, void* stream);
int gemm_tc_splits(const GemmArgs& g);
int gemm_tc_tile_n();
int launch_gemm_simt_f32(const GemmArgs& g, void* stream);
int gemm_simt_tile_n();
int launch_attn_fwd_simt(const gpt_config& c, const void* q, const void* k, const void* v,
                         void* o, float* lse, void* stream);
int launch_attn_fwd_tc(const gpt_config& c, const void* q, const void* k, const void* v, void* o,
                       float* lse, int32_t* status, void* stream);
int launch_attn_bwd_simt(const gpt_config& c, const void* q, const void* k, const void* v,
                         const void* o, const void* dO, const float* lse, const float* rq,
                         const float* rk, const float* cos_t, const float* sin_t, float* Dbuf,
                         void* dqkv, void* stream);

int launch_attn_bwd_tc(const gpt_config& c, const void* q, const void* k, const void* v,
                       const void* o, const void* dO, const float* lse, const float* rq,
                       const float* rk, const float* cos_t, const float* sin_t, float* Dbuf,
                       void* dqkv, float* norm_part, int32_t* status, void* stream);

int launch_gemm(const gpt_config& c, const GemmArgs& g, void* stream) {
  return c.dtype == GPT_BF16 ? launch_gemm_tc(g, stream) : launch_gemm_simt_f32(g, stream);
}

int gemm_kernel_count(const gpt_config& c, const GemmArgs& g) {
  return c.dtype == GPT_BF16 && gemm_tc_splits(g) > 1 ? 2 : 1;
}

int gemm_ce_tile_n(const gpt_config& c) {
  return c.dtype == GPT_BF16 ? gemm_tc_tile_n() : gemm_simt_tile_n();
}

int launch_attn_fwd(const gpt_config& c, const void* q, const void* k, const void* v, void* o,
                    float* lse, int32_t* status, void* stream) {
  return c.dtype == GPT_BF16 ? launch_attn_fwd_tc(c, q, k, v, o, lse, status, stream)
                             : launch_attn_fwd_simt(c, q, k, v, o, lse, stream);
}

int launch_attn_bwd(const gpt_config& c, const void* q, const void* k, const void* v,
                    const void* o, const void* dO, const float* lse, const float* rq,
                    const float* rk, const float* cos_t, const float* sin_t, float* Dbuf,
                    void* dqkv, float* norm_part, int32_t* status, void* stream) {
  if (c.dtype != GPT_BF16 && norm_part) return 1;  // the row partials are a tensor-core output
  return c.dtype == GPT_BF16
             ? launch_attn_bwd_tc(c, q, k, v, o, dO, lse, rq, rk, cos_t, sin_t, Dbuf, dqkv, norm_part,
                                  status, stream)
             : launch_attn_bwd_simt(c, q, k, v, o, dO, lse, rq, rk, cos_t, sin_t, Dbuf, dqkv,
                                    stream);
}

}  // namespace gpt
