// Library-internal helpers shared between translation units (not part of the ABI).
#pragma once

// Records `fmt` as this thread's tq_last_error() message and returns `code`.
__attribute__((visibility("hidden"))) int tq_internal_fail(int code, const char* fmt, ...);
