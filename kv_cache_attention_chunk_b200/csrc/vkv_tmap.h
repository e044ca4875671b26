// Tensor-map encoding with a selectable swizzle (vkv_common.cu).
#pragma once

#include "vkv_internal.h"

namespace vkv {

// As encode_tmap_bf16_4d, with swizzle_bytes 128 (box rows of 128 B) or 64
// (box rows of 64 B); false for any other value or when encoding fails.
bool encode_tmap_bf16_4d_swizzle(CUtensorMap* tm, const void* ptr, const uint64_t dims[4],
                                 const uint64_t strides_bytes[3], const uint32_t box[4], int swizzle_bytes);

}  // namespace vkv
