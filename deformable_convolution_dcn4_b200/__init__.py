"""B200-native (sm_100a) DCNv4 deformable spatial aggregation and the FlowDCN
groupwise multi-scale variant, behind a small C ABI (include/dcn4.h).

The Python names mirror the C entry points; see _binding for arguments.
"""
from ._binding import (Dcn4Error, dcn4_backward, dcn4_backward_noalloc,
                       dcn4_backward_workspace_size, dcn4_forward,
                       dcn4_forward_workspace_size, dcn4_fused_forward,
                       dcn4_fused_forward_workspace_size, dcn4_kernel_launches,
                       dcn4_last_device_error, dcn4_offset_producer, dcn4_out_shape,
                       dcn4_status_string, load, make_desc, msdcn_backward, msdcn_forward)

__all__ = ["Dcn4Error", "dcn4_backward", "dcn4_backward_noalloc", "dcn4_backward_workspace_size",
           "dcn4_forward", "dcn4_forward_workspace_size", "dcn4_fused_forward",
           "dcn4_fused_forward_workspace_size",
           "dcn4_kernel_launches", "dcn4_last_device_error", "dcn4_offset_producer",
           "dcn4_out_shape", "dcn4_status_string", "load", "make_desc", "msdcn_backward",
           "msdcn_forward"]
