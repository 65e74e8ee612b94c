// Dense causal GQA prefill (the baseline the pages compare MSA against).
#include "internal.h"

namespace msa {

cudaError_t launch_dense_prefill(const msa_shape&, const uint16_t*, const uint16_t*,
                                 const uint16_t*, uint16_t*, float*, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace msa
