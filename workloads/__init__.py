"""Seeded synthetic inputs shared by the oracle tests, the CUDA tests and the benchmark."""
from .gen import (BASE_SEED, CONFIG_NAMES, FeistelPermutation, Workload, build_workload,
                  config_workload, draw_cores, near_cubic_factors, random_workload, sub_batch,
                  table_rows_log_uniform, zipf_ranks)

__all__ = ["BASE_SEED", "CONFIG_NAMES", "FeistelPermutation", "Workload", "build_workload",
           "config_workload", "draw_cores", "near_cubic_factors", "random_workload", "sub_batch",
           "table_rows_log_uniform", "zipf_ranks"]
