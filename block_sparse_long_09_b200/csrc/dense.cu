// dense.cu -- dense causal GQA attention baseline (placeholder until the tcgen05 version lands).
#include "kernels.cuh"

namespace qsa {

cudaError_t launch_dense_attn(const DenseArgs &a, cudaStream_t stream)
{
    (void)a;
    (void)stream;
    return cudaErrorNotSupported;
}

}  // namespace qsa
