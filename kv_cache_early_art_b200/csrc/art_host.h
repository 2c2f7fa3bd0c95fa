// art_host.h -- host-side argument-check helpers shared by the entry points.
#pragma once

#include <cstdint>

#include "../../include/art.h"

namespace art_host {

inline bool is_null(const art_tensor_t *t) { return t == nullptr || t->data == nullptr; }

inline int64_t elem_size(int32_t dt) { return dt == ART_BF16 ? 2 : 4; }

inline bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// The smallest workspace (a ring of 16 block states per unit) with which
// art_decode_attention_ex runs p with merge_cta = 2, whatever p's merge_cta
// and workspace hold; a negative art_status_t when the arguments are invalid
// or that walk is not built for them.  Nothing is launched.
int64_t gr_min_workspace_bytes(const art_params_t *p);

}  // namespace art_host
