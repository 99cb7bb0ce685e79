// Step 4 of the DHSA path for bf16 inputs: the launch dispatch by head
// dimension, and the TMA view of the packed token tensors that every bf16
// attention kernel reads through.
//
// out[t, h] = sum_s softmax_s(q[t,h] . k[s,g] * scale) v[s,g] over the kept
// key tokens s <= t, i.e. the tokens of the chunks in plan row (h, chunk(t))
// ("Long-Context Modeling with Dynamic Hierarchical Sparse Attention for
// On-Device LLMs", Abstract: only the token-level interactions selected by the
// upsampled chunk scores are preserved; "... for Memory-Constrained LLM
// Inference": causally important dependencies are kept).
//   head_dim 64, 128: attention_bf16_pair.cu (two query tiles per work item,
//                     persistent CTAs)
//   head_dim 256:     attention_bf16_d256.cu (one query tile per CTA)
#include "common.cuh"
#include "launchers.h"

namespace dhsa {

// 3-D (d, heads, tokens) view of a packed THD bf16 tensor with a (64, 1,
// box_rows) box and 128-byte swizzle: one box lands as box_rows x 128 bytes,
// the canonical K-major SW128 operand layout of tcgen05.mma.
CUresult encode_qkv_map(CUtensorMap* map, const void* base, int heads, int head_dim, int tokens, int box_rows,
                        bool f16) {
  using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
  static EncodeFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || p == nullptr)
      return CUDA_ERROR_NOT_FOUND;
    fn = reinterpret_cast<EncodeFn>(p);
  }
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(heads),
                              static_cast<cuuint64_t>(tokens)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(head_dim) * 2,
                                 static_cast<cuuint64_t>(heads) * head_dim * 2};
  const cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

cudaError_t launch_attention_bf16(const AttnBf16Args& a, cudaStream_t stream) {
  if (a.total_tokens <= 0 || a.num_chunks <= 0) return cudaSuccess;
  switch (a.head_dim) {
    case 64:
    case 128:
      return launch_attention_pair(a, stream);  // two query tiles per CTA (attention_bf16_pair.cu)
    case 256:
      return launch_attention_d256(a, stream);  // attention_bf16_d256.cu
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace dhsa
