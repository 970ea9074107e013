// Library-internal helpers shared between translation units (not part of the ABI).
#pragma once

// Records `fmt` as this thread's tq_last_error() message and returns `code`.
__attribute__((visibility("hidden"))) int tq_internal_fail(int code, const char* fmt, ...);

#include <stddef.h>
#include <stdint.h>
struct tq_handle;
// Workspace bytes tq_attn_decode needs at least (tq_attn_workspace_bytes may ask for more: the
// scores buffer of the two-kernel attention, used only when the workspace holds it).
extern "C" __attribute__((visibility("hidden"))) size_t tq_internal_attn_workspace_min_bytes(
    const tq_handle* hk, const tq_handle* hv, int B, int Hq, int Hkv, int64_t L_cap);
