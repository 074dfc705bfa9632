// Host helpers shared by the library's translation units.
#pragma once
#include <cstdarg>
#include <cstdio>

#include "pa.h"

namespace pa {

// Records a message for pa_last_error() (thread-local) and returns `st`.
pa_status fail(pa_status st, const char* fmt, ...);
void clear_error();

}  // namespace pa
