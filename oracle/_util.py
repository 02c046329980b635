"""Input conversion shared by the oracle modules."""
import numpy as np


def as64(x):
    """Any array-like (numpy, or a torch tensor of any dtype) -> float64 numpy."""
    if hasattr(x, "detach"):
        return x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)
