// gad_error.h - the library's one error-message store, shared by its
// translation units (not part of the public interface).
#pragma once

// Sets the message gad_last_error() returns on this host thread (printf-style)
// and returns `status`.
__attribute__((visibility("hidden"))) int gad_fail(int status, const char* fmt, ...)
    __attribute__((format(printf, 2, 3)));
