"""Seeded synthetic inputs for few-bit KV-cache decode attention.

This module holds NO arithmetic of the method itself: it draws random numbers and builds
synthetic tensors. It is the one module that both the product path (through its tests and
bench) and the CPU oracle consume, so that both see identical inputs:

* the method's own random draws -- the rotation's +-1 sign diagonal and the QJL Gaussian
  matrix -- from a counter-based generator defined here (splitmix64 finaliser over a Weyl
  sequence, Box-Muller for normals), which both sides receive as plain arrays;
* synthetic K/V/query tensors shaped like the workloads the pages discuss (GQA decode layers
  of an 8B- and a 70B-class model, a 1-bit large-batch case, and an MLA-style latent cache),
  drawn with torch's seeded generators on whatever device the caller names.
"""
from .rng import splitmix64, uniform53, rotation_signs, qjl_matrix  # noqa: F401
from .workloads import WORKLOADS, VARIANTS, Workload, get_workload, generate  # noqa: F401
