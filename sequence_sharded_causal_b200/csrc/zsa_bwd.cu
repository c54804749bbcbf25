// zsa_bwd.cu -- backward kernels (K2 preprocess, K3 main, K4 dQ epilogue).
#include "zsa_kernels.h"

namespace zsa {

int launch_bwd(const BwdArgs&, cudaStream_t) { return int(cudaErrorNotSupported); }

}  // namespace zsa
