/* A plain C99 caller of the library's C ABI: compiled and linked (not run)
 * by tests/test_c_abi_user.py, so the header stays usable from C and every
 * entry point the header declares resolves in libbitssm.so. */
#include <stdio.h>

#include "bitssm.h"

typedef void (*entry_fn)(void);

int main(void) {
  bitssm_layer layer = {0};
  size_t bytes = 0;
  unsigned int flags = 0;
  long bad = 0;
  const uint8_t packed[2] = {0x55, 0x55};
  /* host-only calls: no device is touched */
  printf("abi %d, %s\n", bitssm_version(), bitssm_status_string(BITSSM_ERR_WORKSPACE));
  if (bitssm_check_packed(packed, 1, 8, &bad) != BITSSM_OK || bad != 0) return 1;
  if (bitssm_workspace_size(&layer, 1, 1, BITSSM_BF16, BITSSM_A8, &bytes) != BITSSM_ERR_INVALID_ARG)
    return 2;
  /* the device entry points, referenced so the link resolves them */
  entry_fn const entry[] = {
      (entry_fn)bitssm_forward, (entry_fn)bitssm_forward_state, (entry_fn)bitssm_step,
      (entry_fn)bitssm_stack_forward, (entry_fn)bitssm_forward_host,
      (entry_fn)bitssm_forward_timed, (entry_fn)bitlinear_forward,
      (entry_fn)bitlinear_forward_noalloc, (entry_fn)selective_scan_forward,
      (entry_fn)ssd_scan_forward, (entry_fn)bitssm_pack_ternary,
      (entry_fn)bitssm_prepare_weights, (entry_fn)bitssm_device_error,
      (entry_fn)bitssm_selftest_wait, (entry_fn)bitssm_workspace_layout};
  (void)flags;
  return entry[0] != NULL ? 0 : 3;
}
