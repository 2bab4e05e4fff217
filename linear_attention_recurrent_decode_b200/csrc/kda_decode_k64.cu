// kda_decode_k64.cu -- the decode kernels for K = 64 (one translation unit per
// K so that the library compiles in parallel; see kda_decode_pick.cuh).
#include "kda_decode_pick.cuh"

namespace kda {
template cudaError_t pick_decode_kernel<64>(const KernelChoice&, const void**, int*);
}  // namespace kda
