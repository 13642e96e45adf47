/*
 * fa_test_hooks.h -- the extra entry point of the watchdog TEST library,
 * libfa_testhooks.so, which is built from the same sources as libfa.so with
 * FA_TEST_HOOKS defined and a 10 ms device wait limit (FA_WAIT_LIMIT_NS),
 * for the fp16 head dims 64 and 128 only.  libfa.so itself has no hooks and
 * does not export this symbol.  The pages have no counterpart: it exists to
 * show on the GPU that the kernels' bounded waits end a launch cleanly when
 * a copy never arrives.
 */
#ifndef FA_TEST_HOOKS_H
#define FA_TEST_HOOKS_H

#ifdef __cplusplus
extern "C" {
#endif

/*
 * fa_test_set_withhold -- from the next forward launch on, the K/Q producer
 * warp of CTA 0 skips the copy of key block `block` (an index of 128-key
 * blocks; -1 restores normal operation).  The MMA warp's wait for that
 * block then gives up after the wait limit, raises the CTA's abort flag and
 * the device status word; every role leaves its loop, the producers let
 * their copies in flight land, the MMA warp waits for its issued MMAs, TMEM
 * is freed and the launch ends.  fa_get_device_status() then returns
 * FA_ERR_TIMEOUT (once) and the outputs of that launch are not valid.
 * Returns FA_OK or FA_ERR_CUDA (the device symbol could not be written).
 */
int fa_test_set_withhold(int block);

#ifdef __cplusplus
}
#endif

#endif /* FA_TEST_HOOKS_H */
