"""B200 (sm_100a) CUDA library for the Mamba-2 SSD mixer core of Nemotron-H hybrids.

The compute lives in ``libssd_mixer.so`` (C ABI: include/ssd_mixer.h). This package
holds the kernels' sources (csrc/), the build script, the ctypes binding
(:mod:`.ssd_mixer`) and the seeded synthetic workloads (:mod:`.workloads`).
Importing the package does not load the library; the first call does.
"""
from .ssd_mixer import (Dims, SsdError, alloc_workspace, backward, decode_step, load_library, prefill,  # noqa: F401
                        ssd_mixer_backward, ssd_mixer_backward_workspace_size, ssd_mixer_decode_step,
                        ssd_mixer_prefill, ssd_mixer_prefill_state, ssd_mixer_prefill_varlen,
                        ssd_mixer_prefill_workspace_size, ssd_mixer_state_pass, ssd_mixer_workspace_status)
