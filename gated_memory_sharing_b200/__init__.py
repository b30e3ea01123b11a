"""SambaY scan + Gated Memory Unit hot path on B200 (sm_100a).

The product is the C-ABI library ``lib/libsambay.so`` (see ``include/sambay.h``);
:mod:`.abi` is its ctypes binding, :mod:`.layers` keeps weights and workspaces
on the device, :mod:`.synth` generates the seeded synthetic workloads, and
:mod:`.build` compiles the library.  Importing this package loads nothing.
"""

__version__ = "0.1.0"
