"""Seeded synthetic inputs for the DLRM hot path.

Shared by the oracle tests and the CUDA path as the one source of inputs. It
holds input generation only: no pooling, interaction, MLP or loss arithmetic.
"""
from .configs import CONFIGS, Config, ld_pad, shrink  # noqa: F401
from . import gen  # noqa: F401
