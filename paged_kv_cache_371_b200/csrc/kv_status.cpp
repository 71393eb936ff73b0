#include <string>

#include "../../include/paged_kv.h"
#include "kv_status.h"

namespace {
thread_local std::string g_last_error;
}

int kv_fail(int code, const char* msg)
{
    g_last_error = msg ? msg : "";
    return code;
}

void kv_clear_error() { g_last_error.clear(); }

extern "C" const char* kv_last_error_string(void) { return g_last_error.c_str(); }
