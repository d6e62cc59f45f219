// Host-side helpers shared by the entry points of liblsa: argument checks,
// per-device launch facts and the driver's tensor-map encoder.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "../../include/lsa.h"

namespace lsa {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Number of SMs of the current device (cached per device), or -1 without a device.
int device_sm_count();

// Records the last CUDA error as LSA_ERR_CUDA (clearing it), or returns LSA_OK.
int launch_status();

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime
// (the library does not link libcuda directly, so it loads on machines
// without a driver).  Returns nullptr when the driver is unavailable.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);
EncodeTiledFn tensor_map_encoder();

// Launches `kernel` as a programmatic dependent launch on `s`: its grid may be
// launched once every CTA of the previous kernel on the stream has signalled
// griddepcontrol.launch_dependents, so its launch latency overlaps that
// kernel's run.  Every kernel launched this way executes griddepcontrol.wait
// before its first global-memory access (except the reads that a caller's
// flag declares settled: LSA_ATTN_KV_UNCHANGED, LSA_TOKENS_UNCHANGED), which
// orders it after the previous kernel's completion and memory flush; its
// loads after the wait are plain (ld_dep), never non-coherent; and every CTA
// that ends early waits first, so the grid never completes before the one it
// depends on.
//
// With pdl == false it is an ordinary stream-ordered launch (the griddepcontrol
// instructions are then no-ops).  The kernels of the per-step chain use PDL;
// the once-per-window kernels do not: there, the next grid's CTAs waiting on
// the SMs slowed the running selection more than the hidden launch saved.
template <typename... KArgs, typename... Args>
inline void launch_pdl(bool pdl, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

namespace score {
// The token scorer's launch (lsa_index_score.cu); with hist != nullptr it also
// adds each sequence's score-bin counts to hist[b][kScoreBins].
int launch_token_score(const void* q_idx, const float* w, const void* token_keys, int64_t n_slots,
                       const int32_t* chunk_table, const int32_t* kept, const int32_t* n_kept, int B, int max_chunks,
                       int max_kept, float* scores, int32_t* n_tokens, int32_t* hist, int keys_unchanged,
                       cudaStream_t stream);
}  // namespace score

}  // namespace lsa

unsigned* lsa_device_status_ptr();
