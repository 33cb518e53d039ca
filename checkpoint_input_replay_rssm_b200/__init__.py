"""Replay-based SSM decode state for B200: checkpoint + low-precision read copy +
input ring buffer, with hand-written sm_100a kernels behind a C ABI (librssm.so).

Importing the package loads nothing; ``checkpoint_input_replay_rssm_b200.rssm``
is the ctypes binding of the C ABI and ``inputs`` the seeded synthetic inputs.
"""
