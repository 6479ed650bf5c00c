"""CPU checks of the C ABI: the library loads, exports every function declared
in include/kvq.h, and its host-side logic (status strings, memory formula,
split planner, argument validation) behaves as documented.  No kernel is
launched here."""
import ctypes
import os
import re

import pytest
import torch

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kvq.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(kvq_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


@pytest.fixture(scope="module")
def kvq():
    import decode_attention_kvq_b200 as m
    return m


def test_header_declares_the_four_calls():
    names = _declared_functions()
    for n in ("kvq_append", "kvq_append_paged", "kvq_decode_attn", "kvq_dequant"):
        assert n in names


def test_library_exports_every_declared_symbol(kvq):
    lib = ctypes.CDLL(kvq.LIB_PATH)
    missing = [n for n in _declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings_and_version(kvq):
    for code, name in [(0, "KVQ_OK"), (1, "KVQ_ERR_INVALID_ARG"), (2, "KVQ_ERR_UNSUPPORTED"),
                       (3, "KVQ_ERR_CUDA"), (4, "KVQ_ERR_DEVICE_FLAG")]:
        assert kvq.lib.kvq_status_string(code).decode() == name
    assert "sm_100a" in kvq.kvq_version()


@pytest.mark.parametrize("mode,grp", [("per_token", 128), ("group32", 32)])
def test_cache_bytes_matches_oracle_formula(kvq, mode, grp):
    for (L, Hk, S, D) in [(32, 8, 4096, 128), (1, 1, 257, 64), (3, 2, 100, 64)]:
        g = D if mode == "per_token" else grp
        assert kvq.kvq_cache_bytes(L, Hk, S, D, mode) == oracle.cache_bytes(L, Hk, S, D, g)


@pytest.mark.parametrize("B,Hk,hint,ns", [(1, 8, 4097, 0), (16, 8, 8193, 0), (32, 8, 16385, 0),
                                          (1, 8, 131073, 0), (1, 1, 257, 0), (1, 1, 5, 0),
                                          (2, 2, 1000, 7), (1, 1, 33, 100), (4, 2, 0, 0),
                                          (1, 1, 10_000_000, 0)])
def test_decode_plan_covers_hint(kvq, B, Hk, hint, ns):
    chunk, splits = kvq.kvq_decode_plan(B, Hk, hint, ns, num_sms=148)
    assert chunk >= 16 and chunk % 16 == 0
    assert 1 <= splits <= 4096
    assert splits * chunk >= hint
    assert (splits - 1) * chunk < max(hint, 1)          # no empty trailing split
    if ns:
        assert splits <= ns


def test_decode_plan_fills_the_machine(kvq):
    # few (sequence, kv head) units: one equal chunk per CTA, at most one per SM
    chunk, splits = kvq.kvq_decode_plan(1, 8, 4097, 0, num_sms=148)
    assert (chunk, splits) == (240, 18) and 8 * splits <= 148
    chunk, splits = kvq.kvq_decode_plan(1, 8, 131073, 0, num_sms=148)
    assert (chunk, splits) == (7296, 18) and 8 * splits <= 148
    # many units: one-stage (128-token) chunks balance the CTAs' blocks
    chunk, splits = kvq.kvq_decode_plan(37, 8, 16385, 0, num_sms=148)
    assert chunk == 128 and splits == -(-16385 // 128)
    chunk, splits = kvq.kvq_decode_plan(16, 8, 8193, 0, num_sms=148)
    assert chunk == 128 and splits == 65
    # the split count stays bounded for very long caches
    chunk, splits = kvq.kvq_decode_plan(64, 8, 10_000_000, 0, num_sms=148)
    assert splits <= 4096 and chunk % 16 == 0
    # explicit split counts are honoured up to the 16-token rounding of the chunk
    chunk, splits = kvq.kvq_decode_plan(1, 8, 4097, 64, num_sms=148)
    assert 16 < splits <= 64


def test_decode_plan_keeps_short_sequences_whole(kvq):
    # few units and at most four 128-token stages: one chunk, no combine
    assert kvq.kvq_decode_plan(1, 1, 257, 0, num_sms=148) == (272, 1)
    assert kvq.kvq_decode_plan(2, 2, 512, 0, num_sms=148) == (512, 1)
    # one token more: split over the SMs again
    chunk, splits = kvq.kvq_decode_plan(1, 1, 513, 0, num_sms=148)
    assert splits > 1 and splits * chunk >= 513
    # many units keep one-stage chunks whatever the length
    assert kvq.kvq_decode_plan(64, 8, 300, 0, num_sms=148) == (128, 3)
    # an explicit split count still splits a short sequence
    assert kvq.kvq_decode_plan(1, 1, 257, 4, num_sms=148)[1] == 4


def test_workspace_formula(kvq):
    if torch.cuda.is_available():
        pytest.skip("formula check uses an explicit SM count; covered on the GPU")
    # the ABI sizes the workspace from the same plan: B*Hq*splits*(D+2) floats
    chunk, splits = kvq.kvq_decode_plan(1, 8, 4097, 0, num_sms=148)
    assert splits > 1


needs_no_gpu = pytest.mark.skipif(torch.cuda.is_available(),
                                  reason="fake-pointer validation checks run only without a GPU")

FAKE = 4096          # aligned, non-null, never dereferenced: every call below is rejected first


@needs_no_gpu
def test_append_rejects_bad_arguments(kvq):
    lib = kvq.lib
    args = [FAKE, FAKE, 1, 8, 1, 128, 0, FAKE, FAKE, FAKE, FAKE, FAKE, 16, None, None]

    def call(**over):
        a = list(args)
        names = ["k", "v", "B", "Hk", "T", "D", "mode", "pos", "kc", "vc", "ks", "vs",
                 "max_seq", "err", "s"]
        for k2, val in over.items():
            a[names.index(k2)] = val
        return lib.kvq_append(*a)
    assert call(k=None) == 1
    assert call(pos=None) == 1
    assert call(D=72) == 1                  # not a multiple of 16
    assert call(D=512) == 1
    assert call(D=48, mode=1) == 1          # group-32 needs D % 32 == 0
    assert call(B=0) == 1
    assert call(T=0) == 1
    assert call(mode=7) == 1
    assert call(k=FAKE + 2) == 1            # misaligned vector source
    assert call(ks=FAKE + 4) == 1           # scale arrays need 16-byte alignment
    assert call(max_seq=0) == 1


@needs_no_gpu
def test_append_paged_requires_page_size_16(kvq):
    lib = kvq.lib
    base = [FAKE, FAKE, 1, 8, 1, 128, 0, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 4]
    assert lib.kvq_append_paged(*base, 32, None, None) == 1
    assert lib.kvq_append_paged(*base[:12], None, 4, 4, 16, None, None) == 1


@needs_no_gpu
def test_decode_rejects_bad_arguments(kvq):
    lib = kvq.lib
    cv = kvq.CacheView(FAKE, FAKE, FAKE, FAKE, 0, 4096, 0, 0, 0)
    ok = dict(q=FAKE, B=1, Hq=32, Hk=8, D=128, mode=0, kv=ctypes.byref(cv), sl=FAKE, hint=4096,
              scale=0.088, out=FAKE, ws=FAKE, wsb=1 << 30, ns=0, err=None, s=None)

    def call(**over):
        a = dict(ok)
        a.update(over)
        return lib.kvq_decode_attn(*a.values())
    assert call(q=None) == 1
    assert call(Hq=30) == 1                 # Hq % Hk != 0
    assert call(D=100) == 1
    assert call(mode=1, D=48) == 1
    # shapes outside the tensor-core kernels (other head dims, more than 16
    # rows per kv head outside the dense kernel, more than 1024 sequences) are
    # accepted for the CUDA-core kernel: validation passes and the call stops
    # at the device query, which fails here without a GPU (KVQ_ERR_CUDA)
    assert call(D=256) == 3
    assert call(D=32) == 3
    assert call(D=48) == 3
    assert call(Hq=8 * 32, Hk=8, D=64) == 3
    assert call(Hq=8 * 32, Hk=8, mode=1) == 3
    assert call(B=1025) == 3
    assert call(out=FAKE + 4) == 1          # misaligned output
    cv_bad_scale = kvq.CacheView(FAKE, FAKE, FAKE + 8, FAKE, 0, 4096, 0, 0, 0)
    assert call(kv=ctypes.byref(cv_bad_scale)) == 1
    assert call(hint=-1) == 1
    bad_page = kvq.CacheView(FAKE, FAKE, FAKE, FAKE, 32, 0, FAKE, 4, 4)
    assert call(kv=ctypes.byref(bad_page)) == 1
    no_table = kvq.CacheView(FAKE, FAKE, FAKE, FAKE, 16, 0, None, 4, 4)
    assert call(kv=ctypes.byref(no_table)) == 1


@needs_no_gpu
def test_append_decode_rejects_bad_arguments(kvq):
    lib = kvq.lib
    cv = kvq.CacheView(FAKE, FAKE, FAKE, FAKE, 0, 4096, 0, 0, 0)
    ok = dict(q=FAKE, kn=FAKE, vn=FAKE, B=1, Hq=32, Hk=8, D=128, mode=0, kv=ctypes.byref(cv),
              sl=FAKE, hint=4096, scale=0.088, out=FAKE, ws=FAKE, wsb=1 << 30, ns=0, err=None,
              s=None)

    def call(**over):
        a = dict(ok)
        a.update(over)
        return lib.kvq_append_decode(*a.values())
    assert call(kn=None) == 1
    assert call(vn=None) == 1
    assert call(vn=FAKE + 2) == 1           # misaligned new values
    assert call(q=None) == 1
    assert call(mode=9) == 1
    for m in (2, 3, 4, 5):                  # FP8, per-head, per-channel: not fused
        assert call(mode=m) == 2
    assert call(Hq=30) == 1
    # any head dim and group size (the CUDA-core kernel): past validation
    assert call(Hq=8 * 32) == 3
    assert call(D=256) == 3


@needs_no_gpu
def test_error_word_helpers_reject_bad_pointers(kvq):
    assert kvq.lib.kvq_read_error(None, None, None) == 1
    assert kvq.lib.kvq_check_error(None, None) == 1
    assert kvq.lib.kvq_check_error(FAKE + 2, None) == 1      # misaligned word


@needs_no_gpu
def test_chunk_rejects_bad_arguments(kvq):
    lib = kvq.lib
    cv = kvq.CacheView(FAKE, FAKE, FAKE, FAKE, 0, 4096, 0, 0, 0)
    ok = dict(q=FAKE, B=1, Hq=32, Hk=8, T=4, D=128, mode=0, kv=ctypes.byref(cv), sl=FAKE,
              hint=4096, scale=0.088, out=FAKE, ws=FAKE, wsb=1 << 30, ns=0, err=None, s=None)

    def call(**over):
        a = dict(ok)
        a.update(over)
        return lib.kvq_chunk_attn(*a.values())
    assert call(T=0) == 1
    assert call(q=None) == 1
    # more than 16 rows per kv head outside the dense kernel's shapes (head_dim
    # 128, per-token, contiguous, no window): accepted for the CUDA-core kernel
    # (the call then stops at the device query: no GPU here)
    assert call(T=5, D=64) == 3             # (Hq / Hk) * T = 20 rows per kv head
    assert call(Hq=64, T=3, mode=1) == 3    # 24 rows, group-32 scales
    pv = kvq.CacheView(FAKE, FAKE, FAKE, FAKE, 16, 0, FAKE, 4, 4)
    assert call(T=5, kv=ctypes.byref(pv)) == 3     # paged
    assert call(out=FAKE + 4) == 1


def test_chunk_workspace_is_the_decode_workspace_of_the_rows(kvq):
    for B, Hq, Hk, T, D, hint, ns in [(1, 32, 8, 4, 128, 4097, 0), (3, 8, 2, 2, 64, 999, 5),
                                      (16, 32, 8, 1, 128, 8193, 0)]:
        assert kvq.kvq_chunk_workspace_bytes(B, Hq, Hk, T, D, hint, ns) == \
            kvq.kvq_decode_workspace_bytes(B, Hq * T, Hk, D, hint, ns)
    assert kvq.kvq_chunk_workspace_bytes(1, 32, 8, 0, 128, 4097, 0) == 0
    # above 16 rows per kv head: sized for the CUDA-core kernel too
    assert kvq.kvq_chunk_workspace_bytes(1, 32, 8, 5, 128, 4097, 0) == \
        kvq.kvq_decode_workspace_bytes(1, 32 * 5, 8, 128, 4097, 0)


@needs_no_gpu
def test_dequant_rejects_bad_arguments(kvq):
    lib = kvq.lib
    assert lib.kvq_dequant(FAKE, FAKE, 10, 24, 0, FAKE, None) == 1
    assert lib.kvq_dequant(FAKE, FAKE, -1, 64, 0, FAKE, None) == 1
    assert lib.kvq_dequant(None, FAKE, 10, 64, 0, FAKE, None) == 1
    assert lib.kvq_dequant(FAKE, FAKE, 0, 64, 0, FAKE, None) == 0    # nothing to do
