"""Seeded synthetic inputs shared by the tests, the benchmark and the smoke check."""
from .paged import PagedKV, paginate
from .planted_gap import (CONFIG_SEED_BASE, PlantedInputs, beta_for_gap,
                          config_seed, output_gradient, planted_gap,
                          planted_gap_kv_inplace)

__all__ = ["CONFIG_SEED_BASE", "PagedKV", "PlantedInputs", "beta_for_gap",
           "config_seed", "output_gradient", "paginate", "planted_gap",
           "planted_gap_kv_inplace"]
