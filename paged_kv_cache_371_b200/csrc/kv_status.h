// Thread-local last-error text shared by the host and device halves of the
// library.
#pragma once

int kv_fail(int code, const char* msg);
void kv_clear_error();
