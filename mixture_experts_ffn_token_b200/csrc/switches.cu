// switches.cu -- the library's runtime switches (MOE_B200_* environment
// variables), read in one pass over the environment at the start of every
// API call instead of one getenv per switch and launch.
#include <cstdlib>
#include <cstring>

#include "kernels.cuh"

extern char** environ;

namespace moe {
namespace {

thread_local Switches t_switches;
thread_local bool t_switches_read = false;

long to_long(const char* v) { return std::strtol(v, nullptr, 10); }

}  // namespace

void refresh_switches() {
  Switches s;
  constexpr char kPrefix[] = "MOE_B200_";
  constexpr size_t kPrefixLen = sizeof(kPrefix) - 1;
  for (char** e = environ; e != nullptr && *e != nullptr; ++e) {
    const char* kv = *e;
    if (std::strncmp(kv, kPrefix, kPrefixLen) != 0) continue;
    const char* name = kv + kPrefixLen;
    const char* eq = std::strchr(name, '=');
    if (eq == nullptr) continue;
    const size_t n = static_cast<size_t>(eq - name);
    const char* v = eq + 1;
    auto is = [&](const char* key) { return std::strlen(key) == n && std::strncmp(name, key, n) == 0; };
    if (is("PDL")) s.pdl = v[0] != '0';
    else if (is("CSR_FUSED")) s.csr_fused = v[0] != '0';
    else if (is("TEST_STALL_CSR_MS")) s.test_stall_csr_ms = to_long(v);
    else if (is("FUSED_GATHER")) s.fused_gather = v[0] == '1';
    else if (is("B_ONE_BOX")) s.b_one_box = v[0] != '0';
    else if (is("CTA_PAIR")) s.cta_pair = v[0] == '2' ? 2 : 1;
    else if (is("TEST_STALL_DOWN_TILES_MS")) s.test_stall_down_ms = to_long(v);
    else if (is("TILE_SCHEDULE")) s.tile_schedule = (v[0] == 'd' || v[0] == 's') ? v[0] : 0;
    else if (is("SINGLE_LAUNCH")) s.single_launch = v[0] != '0';
    else if (is("PDL_COOP")) s.pdl_coop = v[0] != '0';
    else if (is("PAIR_COOP")) s.pair_coop = v[0] != '0';
  }
  t_switches = s;
  t_switches_read = true;
}

const Switches& switches() {
  if (!t_switches_read) refresh_switches();
  return t_switches;
}

}  // namespace moe
