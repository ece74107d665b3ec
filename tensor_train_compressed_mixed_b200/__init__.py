"""B200-native Tensor-Train embedding gather (libttemb + a thin ctypes binding)."""
from . import abi, dp
from .abi import TTEmbError
from .embedding import TTEmbeddingBag, from_workload

__all__ = ["abi", "dp", "TTEmbError", "TTEmbeddingBag", "from_workload"]
