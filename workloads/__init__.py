"""Seeded synthetic workloads for the Mamba mixer core.

This package only draws random numbers and lays them out; it holds none of the
mixer's arithmetic.  Both the fp64 oracle (through the tests) and the CUDA path
(through the tests and the benchmark) take their inputs from here.
"""

from .synth import (  # noqa: F401
    CONFIGS,
    MixerConfig,
    DecodeConfig,
    make_mixer_inputs,
    make_decode_inputs,
    make_mixer_inputs_custom,
    make_decode_inputs_custom,
    make_norm_weights,
    make_projection_weights,
    SsdConfig,
    SSD_CONFIGS,
    make_ssd_inputs,
    make_ssd_inputs_custom,
    M3Config,
    M3_CONFIGS,
    make_m3_inputs,
    make_m3_inputs_custom,
    sample_channels,
    subset_channels,
)
