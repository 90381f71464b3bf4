// Partitioned paged decode attention for 16-token blocks.
#include "paged_attention_kernel.cuh"

namespace pkv {
namespace attn {

template cudaError_t dispatch_partitioned<16>(pkv_dtype, bool, int, int, int, const CUtensorMap&, const CUtensorMap&,
                                               const Params&, dim3, cudaStream_t);

}  // namespace attn
}  // namespace pkv
