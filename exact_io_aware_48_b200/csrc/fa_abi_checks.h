// fa_abi_checks.h -- host-side argument checks shared between translation units of libfa.so (not exported).
#pragma once
#include <cstdint>

namespace fa_abi {

// Every argument check fa_bwd makes before it looks at the workspace: pointers (non-null, 16-byte aligned tensors,
// 4-byte aligned lse and key_lens), shape, dtype, scale, head dim and the block-mask tile count.  Returns an
// fa_status; FA_OK when fa_bwd would go on to check the workspace.
__attribute__((visibility("hidden"))) int bwd_check_args(const void* q, const void* k, const void* v, const void* o,
                                                         const void* dout, const float* lse, const void* dq,
                                                         const void* dk, const void* dv, int B, int H, int N, int d,
                                                         float softmax_scale, const int32_t* key_lens,
                                                         const uint8_t* block_mask, int dtype);

}  // namespace fa_abi
