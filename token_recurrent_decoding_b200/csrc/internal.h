// Library-internal entry points shared between the translation units of
// librlt.so (hidden: not part of the C ABI).
#pragma once

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime.h>

namespace rlt {

// Validates the arguments of the standalone decode attention and runs it
// with the given device workspace (>= its computed size, 256-byte aligned).
int attend_run_internal(const float *q, const void *kv, const int32_t *h_lengths, int n, int H,
                        int dh, int cap, int dtype, void *out, void *workspace,
                        size_t workspace_bytes, cudaStream_t st);

// Workspace bytes of the standalone decode attention (0: invalid shape).
size_t attend_workspace_internal(int n, int H, int dh, int cap);

}  // namespace rlt
