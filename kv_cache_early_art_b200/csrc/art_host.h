// art_host.h -- host-side argument-check helpers shared by the entry points.
#pragma once

#include <cstdint>

#include "../../include/art.h"

namespace art_host {

inline bool is_null(const art_tensor_t *t) { return t == nullptr || t->data == nullptr; }

inline int64_t elem_size(int32_t dt) { return dt == ART_BF16 ? 2 : 4; }

inline bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace art_host
