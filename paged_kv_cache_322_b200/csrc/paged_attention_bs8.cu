// Partitioned paged decode attention for 8-token blocks.
#include "paged_attention_kernel.cuh"

namespace pkv {
namespace attn {

template cudaError_t dispatch_partitioned<8>(pkv_dtype, bool, int, int, int, const CUtensorMap&, const CUtensorMap&,
                                               const Params&, dim3, cudaStream_t);

}  // namespace attn
}  // namespace pkv
