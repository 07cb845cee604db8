// FP8 KV cache decode (656-byte tokens).
#include "mla_internal.h"

namespace mla {

int launch_decode_fp8(const CUtensorMap&, const CUtensorMap&, const DecodeParams&, cudaStream_t) {
  return static_cast<int>(cudaErrorNotSupported);
}

}  // namespace mla
