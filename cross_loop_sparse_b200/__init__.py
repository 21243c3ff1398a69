"""FlashLoop lazy loop-r attention sublayer on B200 (sm_100a).

``cross_loop_sparse_b200.flashloop`` is the ctypes binding of the C ABI
(``include/flashloop.h``); importing it loads ``libflashloop.so`` and fails
loudly when the library has not been built.
"""
