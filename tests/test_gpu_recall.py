"""Parity of the recall kernels (keep mask -> index list -> resident buffer)
with the CPU oracle, bit for bit: several compaction blocks per row with a
ragged tail, masks from empty to full, lists longer and shorter than max_sel,
rows that start on 16 bytes (the mask landed in shared memory by bulk
copies) and rows that do not or are too long for it (register form);
records of 132 B and 1024 B (bulk copies from device memory, also at
sources and strides off the 16-byte grid; 4- and 16-byte loads from pinned
host memory) and 131 B (byte copies)."""
import numpy as np
import pytest
import torch

import oracle.recall as OR

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from learned_kv_chunk_b200 import fm  # noqa: E402  (loads libfm.so; raises if missing)

DEV = torch.device("cuda", 0)


def _masks(B, N, seed):
    g = torch.Generator().manual_seed(seed)
    dens = torch.tensor([0.0, 0.001, 0.02, 0.5, 0.999, 1.0])[:B]
    return (torch.rand(B, N, generator=g) < dens[:, None]).to(torch.uint8)


@pytest.mark.parametrize("N", [3 * 16384 + 77, 2 * 16384 + 32, 2 * 16384 + 48, 5, 16384, 17 * 16384 + 16])
@pytest.mark.parametrize("max_sel", [1, 100, 4096, 70000])
def test_compact_matches_oracle(N, max_sel):
    keep = _masks(6, N, N + max_sel)
    idx, count = fm.fm_compact_mask(keep.to(DEV), max_sel)
    torch.cuda.synchronize()
    want_idx, want_count = OR.compact_mask(keep.numpy(), max_sel)
    np.testing.assert_array_equal(count.cpu().numpy(), want_count)
    np.testing.assert_array_equal(idx.cpu().numpy(), want_idx)


def test_compact_accepts_bool_and_nonzero_bytes():
    keep = _masks(4, 20000, 3)
    idx_b, cnt_b = fm.fm_compact_mask(keep.bool().to(DEV), 512)
    idx_u, cnt_u = fm.fm_compact_mask((keep * 7).to(DEV), 512)  # any nonzero byte counts as kept
    assert torch.equal(idx_b, idx_u) and torch.equal(cnt_b, cnt_u)


@pytest.mark.parametrize("rec", [132, 1024, 131])
@pytest.mark.parametrize("where", ["device", "pinned"])
def test_gather_matches_oracle(rec, where):
    B, n_src, max_sel = 4, 3000, 600
    g = torch.Generator().manual_seed(rec)
    src = torch.randint(0, 256, (B, n_src, rec), generator=g, dtype=torch.uint8)
    keep = _masks(B, n_src, rec + 1)[[2, 3, 0, 1]]  # densities 2 %, 50 %, 0, 0.1 %
    idx, count = fm.fm_compact_mask(keep.to(DEV), max_sel)
    src_in = src.to(DEV) if where == "device" else src.pin_memory()
    dst = torch.full((B, max_sel, rec), 0xA5, dtype=torch.uint8, device=DEV)
    fm.fm_gather_records(src_in, idx, count, dst)
    torch.cuda.synchronize()
    want = OR.gather_records(src.numpy(), idx.cpu().numpy(), count.cpu().numpy(),
                             np.full((B, max_sel, rec), 0xA5, np.uint8))
    np.testing.assert_array_equal(dst.cpu().numpy(), want)


@pytest.mark.parametrize("src_off,pad", [(4, 0), (8, 4), (12, 12)])
def test_gather_off_grid_sources(src_off, pad):
    """Records that start 4, 8 or 12 bytes past a 16-byte boundary, with row
    strides that move the start from row to row: each bulk copy covers the
    record's 16-byte granules and the record is cut out of them."""
    B, n_src, rec, max_sel = 5, 2100, 132, 300
    stride = n_src * rec + pad
    g = torch.Generator().manual_seed(src_off + 16 * pad)
    flat = torch.randint(0, 256, (src_off + B * stride + 16,), generator=g, dtype=torch.uint8)
    keep = _masks(B, n_src, src_off)[[2, 3, 4, 1, 0]]
    idx, count = fm.fm_compact_mask(keep.to(DEV), max_sel)
    flat_d = flat.to(DEV)
    dst = torch.full((B, max_sel, rec), 0x5A, dtype=torch.uint8, device=DEV)
    base = flat_d.data_ptr() + src_off
    assert base % 16 == src_off
    st = fm.lib().fm_gather_records(base, stride, n_src, rec, idx.data_ptr(), count.data_ptr(), B, max_sel,
                                    dst.data_ptr(), max_sel * rec, None)
    assert st == fm.FM_OK
    torch.cuda.synchronize()
    src = np.stack([flat.numpy()[src_off + b * stride: src_off + b * stride + n_src * rec].reshape(n_src, rec)
                    for b in range(B)])
    want = OR.gather_records(src, idx.cpu().numpy(), count.cpu().numpy(), np.full((B, max_sel, rec), 0x5A, np.uint8))
    np.testing.assert_array_equal(dst.cpu().numpy(), want)


def test_gather_rejects_pageable_host_memory():
    src = torch.zeros(1, 10, 16, dtype=torch.uint8)  # not pinned
    idx = torch.zeros(1, 4, dtype=torch.int32, device=DEV)
    cnt = torch.zeros(1, dtype=torch.int32, device=DEV)
    dst = torch.zeros(1, 4, 16, dtype=torch.uint8, device=DEV)
    st = fm.lib().fm_gather_records(src.data_ptr(), 160, 10, 16, idx.data_ptr(), cnt.data_ptr(), 1, 4,
                                    dst.data_ptr(), 64, None)
    assert st == fm.FM_ERR_INVALID_ARG


def test_topk_mask_to_resident_keys_full_size():
    """64 rows x 262144 chunks, top-4096 mask -> index lists -> the kept
    chunks' 132-byte indexer records gathered from device memory; sampled rows
    against the oracle."""
    B, N, K = 64, 262144, 4096
    g = torch.Generator(device=DEV).manual_seed(11)
    ens = torch.rand(B, N, device=DEV, generator=g)
    keep = fm.fm_select_topk(ens, K)
    idx, count = fm.fm_compact_mask(keep, K)
    keys = torch.randint(0, 256, (B, N, 132), device=DEV, dtype=torch.uint8, generator=g)
    dst = fm.fm_gather_records(keys, idx, count)
    torch.cuda.synchronize()
    assert (count == K).all()
    for b in (0, 17, 63):
        want_idx, want_count = OR.compact_mask(keep[b:b + 1].cpu().numpy(), K)
        np.testing.assert_array_equal(idx[b].cpu().numpy(), want_idx[0])
        want = OR.gather_records(keys[b:b + 1].cpu().numpy(), want_idx, want_count,
                                 np.zeros((1, K, 132), np.uint8))
        np.testing.assert_array_equal(dst[b].cpu().numpy(), want[0])
