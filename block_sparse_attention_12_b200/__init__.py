"""B200-native AB-Attention hot path: IBCS selector, SIP planner and gathered
block-sparse forward, hand-written CUDA for sm_100a behind a C ABI
(include/abattn.h).  The Python layer only marshals arguments."""
