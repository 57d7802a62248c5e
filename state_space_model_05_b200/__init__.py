"""B200 (sm_100a) Mamba-2 SSD prefill and decode behind a C ABI.

``binding`` exposes the C entry points (``ssd_prefill``, ``ssd_decode_step``, ``ssd_decode_steps``,
``ssd_decode_step_layers``, ``ssd_decode_steps_layers``, ``ssd_gdn_decode_step``, ``ssd_prefill_workspace_bytes``,
``ssd_device_status``, ``ssd_set_prefill_path``) on
torch tensors;
``inputs`` holds the seeded synthetic input generators.  Importing the package
does not load the CUDA library; the first call does, and fails loudly if it is
missing.
"""
from .binding import (SSDError, decode_layer_table, ssd_decode_step,  # noqa: F401
                      ssd_decode_step_layers, ssd_decode_steps, ssd_decode_steps_layers, ssd_device_status,
                      ssd_gdn_decode_step,
                      ssd_get_prefill_path, ssd_prefill, ssd_prefill_varlen, ssd_prefill_workspace_bytes,
                      ssd_set_prefill_path)

__all__ = ["SSDError", "ssd_prefill", "ssd_decode_step", "ssd_decode_steps", "ssd_decode_step_layers",
           "ssd_decode_steps_layers",
           "decode_layer_table", "ssd_gdn_decode_step", "ssd_prefill_varlen", "ssd_prefill_workspace_bytes",
           "ssd_device_status", "ssd_set_prefill_path", "ssd_get_prefill_path"]
