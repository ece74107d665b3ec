"""B200-native Tensor-Train embedding gather (libttemb + a thin ctypes binding)."""
from . import abi
from .abi import TTEmbError
from .embedding import TTEmbeddingBag, from_workload

__all__ = ["abi", "TTEmbError", "TTEmbeddingBag", "from_workload"]
