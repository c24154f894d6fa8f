// Host-side helpers shared by the library's translation units.  None of this
// is part of the C ABI.
#pragma once
#include <new>

namespace dash {

// Spin limit of the device waits in microseconds: the value set with
// dash_set_spin_limit_us, else DASH_SPIN_LIMIT_US, else 10 s.
long long spin_limit_us();

// The fault armed with dash_inject_fault (0: none), disarmed by this call.
int take_armed_fault();

// The mode set with dash_set_head_interleave (0: the library's choice).
int head_interleave_mode();

// C++ exceptions (std::bad_alloc from a table, a map or a vector sized by the
// caller's arguments) must not cross the C ABI: each entry point that
// allocates on the host returns a status instead.
template <class R, class F>
R no_throw_impl(F&& f, R on_oom, R on_other) {
  try {
    return f();
  } catch (const std::bad_alloc&) {
    return on_oom;
  } catch (...) {
    return on_other;
  }
}
template <class F>
auto no_throw(F&& f, decltype(f()) on_oom, decltype(f()) on_other) -> decltype(f()) {
  return no_throw_impl<decltype(f())>(static_cast<F&&>(f), on_oom, on_other);
}

}  // namespace dash
