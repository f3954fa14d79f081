"""B200 (sm_100a) element-wise recurrence scans over the time axis.

    mingru_scan(k, hx, h0=None)     minGRU, whole sequence (B, T, D)
    mingru_scan_log(k, hx, h0=None) the same, evaluated in log space
    mingru_step(k_t, hx_t, h_prev)  minGRU, one token (B, D)
    minmax_scan(r, s, x0=None)      MinMax neuron, whole sequence (B, T, D)
    mingru_scan_host / minmax_scan_host   the same for CPU tensors, with the
                                    copies to and from the GPU overlapped
    mingru_scan_backward / minmax_scan_backward   gradients of both scans
    mingru_scan_fn / minmax_scan_fn   differentiable (torch.autograd) scans
    mingru_scan_decay(_backward, _fn)  minGRU with time decay of the state
    mingru_projected_scan(x, w, h0) the layer's input projection (tensor cores)
                                    fused with the scan

All three run in the CUDA library ``libsgr.so`` (C ABI:
include/scan_gated_rnns.h); this package only marshals PyTorch tensors into
it.  Build the library with ``python -m scan_gated_rnns_b200.build``.
"""
from ._abi import ScanError
from .autograd import mingru_scan_decay_fn, mingru_scan_fn, minmax_scan_fn
from .host import mingru_scan_host, minmax_scan_host, staging_size
from .ops import (Workspace, default_workspace, mingru_scan, mingru_scan_backward,
                  mingru_projected_scan, mingru_scan_decay, mingru_scan_decay_backward, mingru_scan_log,
                  mingru_step, minmax_scan,
                  minmax_scan_backward, set_kernel_override, set_tile_override, version,
                  workspace_size)

__all__ = ["ScanError", "Workspace", "default_workspace", "mingru_projected_scan", "mingru_scan",
           "mingru_scan_backward",
           "mingru_scan_decay", "mingru_scan_decay_backward", "mingru_scan_decay_fn", "mingru_scan_fn", "mingru_scan_host", "mingru_scan_log", "mingru_step", "minmax_scan",
           "minmax_scan_backward", "minmax_scan_fn", "minmax_scan_host", "set_kernel_override",
           "set_tile_override", "staging_size", "version", "workspace_size"]
