// Partitioned paged decode attention for 64-token blocks.
#include "paged_attention_kernel.cuh"

namespace pkv {
namespace attn {

template cudaError_t dispatch_partitioned<64>(pkv_dtype, bool, int, int, int, const CUtensorMap&, const CUtensorMap&,
                                               const Params&, dim3, cudaStream_t);

}  // namespace attn
}  // namespace pkv
