// tmap.cu -- host helper shared by the TMA kernels: the driver's cuTensorMapEncodeTiled, obtained through
// the runtime's driver entry point so that the library needs no link-time dependency on libcuda.
#include <mutex>

#include "kernels.h"

namespace gdr {

EncodeTiledFn tensor_map_encoder() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        cudaGetLastError();
    });
    return fn;
}

}  // namespace gdr
