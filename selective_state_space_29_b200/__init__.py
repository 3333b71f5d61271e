"""B200-native (sm_100a) selective scan and recurrent state update of the
Mamba selective state-space model.

The compute path is the CUDA library `libmamba_ssm_b200.so` behind the C ABI
of include/mamba_ssm.h; `mamba_ssm` is its Python binding, `workloads` the
seeded synthetic inputs, `build` the in-tree build.  Importing the package
does not load the library; the first call through `mamba_ssm` does.
"""

__all__ = ["mamba_ssm", "workloads", "build"]
