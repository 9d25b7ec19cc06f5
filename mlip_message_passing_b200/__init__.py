"""B200 (sm_100a) channelwise Clebsch-Gordan tensor product and message-passing convolution.

The compute path is the C-ABI library ``libe3b.so`` (declared in ``include/e3b.h``); the thin
PyTorch binding is ``mlip_message_passing_b200.e3b``.  Import it explicitly; the seeded input
generators in ``mlip_message_passing_b200.workloads`` stay importable without a GPU.
"""
