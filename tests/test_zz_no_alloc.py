"""ep_decompress_noalloc, the entry point for callers that cannot allocate device memory (for
instance a plugin inside an inference engine that owns all device memory, or code that must
avoid the synchronisation a cudaMalloc can cause): it keeps the decoder's tables in a static
device array instead of a caller workspace.  Called through the C ABI, its output must equal
the workspace path's (ep_prepare + ep_decompress) and the oracle's bit for bit, on calls in a row with
different streams and table layouts (paired, single-coded, paired), so each call must replace
the previous call's tables.

The file sorts last so that a run stopping at its first failure has already run every other
test; it also passes alone in a fresh process."""
import ctypes as C

import numpy as np
import pytest
import torch

from dit_weight_compression_tile_b200 import binding as B
from dit_weight_compression_tile_b200 import synth

pytestmark = pytest.mark.gpu


def noalloc_decode(d_blob, info, stream):
    out = torch.empty(info.shape, dtype=info.dtype, device=d_blob.device)
    status = torch.zeros(1, dtype=torch.int32, device=d_blob.device)
    rc = B.lib().ep_decompress_noalloc(C.byref(info), d_blob.data_ptr(), out.data_ptr(), info.container_dtype,
                                       status.data_ptr(), stream.cuda_stream)
    assert rc == 0, B.lib().ep_status_string(rc)
    return out, status


def workspace_decode(d_blob, info, stream):
    status = torch.zeros(1, dtype=torch.int32, device=d_blob.device)
    work = B.prepare(d_blob, info, status=status, stream=stream)
    out = B.decompress(d_blob, info, workspace=work, status=status, stream=stream)
    return out, status


def test_noalloc_matches_workspace_path_twice(oracle):
    # a paired stream (108,544 bytes of tables) then a single-coded one (57,344 bytes) and a paired
    # one again: each call must leave its own tables in the shared array, whatever the one before
    cases = [(synth.row_lognormal(512, 2048, 21), 4.0, 0, B.CODING_PAIRED),
             (synth.gaussian(256, 1024, 0.02, 22), 3.0, B.INT8, B.CODING_SINGLE),
             (synth.gaussian(256, 1024, 0.02, 23), 3.0, B.FP8E4M3, B.CODING_PAIRED)]
    stream = torch.cuda.Stream()
    layouts = []
    for w, target, container, coding in cases:  # calls in a row, each with other tables
        blob = B.compress(w, target, container=container, coding=coding)
        info = B.stream_info(blob)
        layouts.append((info.paired, info.workspace_nbytes))
        d = blob.cuda()
        with torch.cuda.stream(stream):
            got, st_got = noalloc_decode(d, info, stream)
            ref, st_ref = workspace_decode(d, info, stream)
        stream.synchronize()
        assert int(st_got.item()) == 0 and int(st_ref.item()) == 0
        assert got.dtype == ref.dtype and got.shape == ref.shape
        assert np.array_equal(got.view(torch.uint8).cpu().numpy(), ref.view(torch.uint8).cpu().numpy())
        # and both equal the oracle's decode of the same stream, byte for byte
        rc, st, _, out_ref = oracle.decode(blob.numpy())
        assert rc == 0 and st == 0
        assert np.array_equal(got.contiguous().view(torch.uint8).cpu().numpy().reshape(-1),
                              out_ref.view(np.uint8).reshape(-1))
    assert layouts == [(1, 108544), (0, 57344), (1, 108544)]


def test_noalloc_rejects_oversized_workspace():
    blob = B.compress(synth.gaussian(64, 256, 0.02, 23), 4.0)
    info = B.stream_info(blob)
    info.workspace_nbytes = 108544 + 16  # beyond the static array's stated maximum
    d = blob.cuda()
    out = torch.empty(info.shape, dtype=info.dtype, device="cuda")
    rc = B.lib().ep_decompress_noalloc(C.byref(info), d.data_ptr(), out.data_ptr(), info.container_dtype, None,
                                       torch.cuda.current_stream().cuda_stream)
    assert rc == -8  # EP_ERR_UNSUPPORTED
