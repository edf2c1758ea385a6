"""Process-pool tasks of the parity tests (numpy and the oracle only, so a
spawned worker starts without torch or the CUDA library)."""
import numpy as np

from oracle import moe_oracle as O


def abs_wd_times(task):
    """dev @ |Wd|^T for expert e: task = (experts, e, dev)."""
    experts, e, dev = task
    return dev @ np.abs(O.dequant_nvfp4(*experts.expert(e)[2])).T
