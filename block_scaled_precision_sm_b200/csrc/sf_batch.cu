// sf_batch.cu — transform_sf_ue8m0_batched: the scale-factor transform of a stack of
// same-shaped tensors (the per-expert B scales of a grouped GEMM) in one launch.
//
// Each tensor is packed exactly as transform_sf_ue8m0 packs it (pairs of UE8M0 bytes along K
// in one int16, stored MN-major: "DeepSeek lanza kernels de DeepGEMM para Huawei Ascend 950",
// section "Qué incluye el lanzamiento"); the batch only spares a launch and a DRAM round trip
// per tensor.
#include <cuda_runtime.h>

#include <cstdint>

#include "bsp.h"
#include "internal.h"
#include "sf_transform.cuh"

extern "C" int transform_sf_ue8m0_batched(const void* sf_in, int in_kind, int batch, int mn, int kb, int64_t ld_in,
                                          int64_t batch_stride_in, void* sf_out, int64_t ld_out,
                                          int64_t batch_stride_out, void* stream) {
    using namespace bsp;
    if (!sf_in || !sf_out || batch <= 0 || mn <= 0 || kb <= 0 || (in_kind != 0 && in_kind != 1)) return BSP_ERR_ARG;
    if (ld_in < kb || ld_out < mn) return BSP_ERR_SHAPE;
    const int es = in_kind == 0 ? 4 : 1, words = (kb + 1) / 2;
    const int64_t in_extent = (int64_t)(mn - 1) * ld_in + kb;  // elements of one input tensor
    const int64_t out_extent = (int64_t)words * ld_out;          // words of one output tensor
    if (batch > 1 && (batch_stride_in < in_extent || batch_stride_out < out_extent)) return BSP_ERR_SHAPE;
    if ((ld_out * 2) % 16 || (batch > 1 && (batch_stride_out * 2) % 16) ||
        (reinterpret_cast<uintptr_t>(sf_out) & 15u))
        return BSP_ERR_ALIGN;
    if (in_kind == 0 && (reinterpret_cast<uintptr_t>(sf_in) & 3u)) return BSP_ERR_ALIGN;
    const int64_t zin = batch > 1 ? batch_stride_in : 0, zout = batch > 1 ? batch_stride_out : 0;
    const char* ib = static_cast<const char*>(sf_in);
    const char* ie = ib + ((int64_t)(batch - 1) * zin + in_extent) * es;
    const char* ob = static_cast<const char*>(sf_out);
    const char* oe = ob + ((int64_t)(batch - 1) * zout + out_extent) * 2;
    if (ib < oe && ob < ie) return BSP_ERR_ARG;  // overlapping buffers
    if (batch > 65535 || (kb + kSfTileKB - 1) / kSfTileKB > 65535) return BSP_ERR_UNSUPPORTED;
    int* status = nullptr;
    if (const int rc = detail::status_word(&status)) return rc;
    const SfJob job{sf_in, ld_in, static_cast<uint16_t*>(sf_out), ld_out, mn};
    const bool ok = launch_sf_transform_batched(job, batch, zin * es, zout, in_kind, kb, status,
                                                static_cast<cudaStream_t>(stream));
    detail::note_launch();
    return ok ? BSP_OK : BSP_ERR_CUDA;
}
