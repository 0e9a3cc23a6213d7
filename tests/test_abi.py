"""The C ABI on CPU: the library loads, exports every function include/kda.h
declares, and rejects bad arguments before touching the GPU (validation runs
on the host; none of these calls reaches a CUDA API)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def K():
    from linear_attention_recurrence_11_b200 import build
    build.build()
    from linear_attention_recurrence_11_b200 import kda
    return kda


def declared_functions():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^[A-Za-z_][\w \*]*?\b(kda_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for f in ("kda_forward", "kda_forward_ex", "kda_decode_step", "kda_forward_workspace_size",
              "kda_status_string", "kda_forward_launches", "kda_abi_version"):
        assert f in names


def test_library_exports_every_declared_symbol(K):
    lib = ctypes.CDLL(K.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings(K):
    assert K.kda_status_string(0) == "ok"
    for c in range(1, 7):
        assert K.kda_status_string(c) not in ("ok", "unknown status")
    assert K.kda_status_string(99) == "unknown status"
    assert K.kda_abi_version() >= 1


FAKE = 1 << 20  # a 16-byte aligned non-null address; never dereferenced


def fwd(K, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, S0=None, o=FAKE, S_T=None, B=1, T=64, H=2,
             dk=128, dv=128, chunk=64, dtype=1, cu=None, num_seqs=0, ws=None, ws_bytes=0,
             status=None, stream=None, path=0)
    a.update(kw)
    return K._lib.kda_forward_ex(a["q"], a["k"], a["v"], a["g"], a["beta"], a["S0"], a["o"], a["S_T"],
                                 a["B"], a["T"], a["H"], a["dk"], a["dv"], a["chunk"], a["dtype"],
                                 a["cu"], a["num_seqs"], a["ws"], a["ws_bytes"], a["status"],
                                 a["stream"], a["path"])


def test_forward_rejects_bad_sizes(K):
    assert fwd(K, B=0) == K.KDA_ERR_INVALID_ARG
    assert fwd(K, T=-1) == K.KDA_ERR_INVALID_ARG
    assert fwd(K, H=0) == K.KDA_ERR_INVALID_ARG
    assert fwd(K, dtype=7) == K.KDA_ERR_INVALID_ARG
    assert fwd(K, dk=48) == K.KDA_ERR_UNSUPPORTED
    assert fwd(K, dv=256) == K.KDA_ERR_UNSUPPORTED
    assert fwd(K, chunk=128) == K.KDA_ERR_UNSUPPORTED
    assert fwd(K, chunk=0) == K.KDA_ERR_UNSUPPORTED
    assert fwd(K, path=9) == K.KDA_ERR_INVALID_ARG


def test_forward_rejects_bad_pointers(K):
    for name in ("q", "k", "v", "g", "beta", "o"):
        assert fwd(K, **{name: None}) == K.KDA_ERR_INVALID_ARG, name
    for name in ("q", "k", "v", "g", "beta", "o", "S0", "S_T", "cu", "status"):
        kw = {name: FAKE + 4}
        if name == "cu":
            kw["num_seqs"] = 1
        assert fwd(K, **kw) == K.KDA_ERR_ALIGNMENT, name


def test_forward_varlen_rules(K):
    assert fwd(K, cu=FAKE, num_seqs=0) == K.KDA_ERR_INVALID_ARG
    assert fwd(K, cu=FAKE, num_seqs=2, B=2) == K.KDA_ERR_INVALID_ARG
    # the longest-first schedule needs its workspace; missing or short -> rejected before launch
    for path in (0, 1, 2):
        assert fwd(K, cu=FAKE, num_seqs=8, path=path) == K.KDA_ERR_WORKSPACE
        assert fwd(K, cu=FAKE, num_seqs=8, ws=FAKE, ws_bytes=16, path=path) == K.KDA_ERR_WORKSPACE


def test_tc_path_only_where_built(K):
    # fp32 never takes the tensor-core kernel
    assert fwd(K, dtype=0, path=K.PATHS["tc"]) == K.KDA_ERR_UNSUPPORTED
    assert fwd(K, dk=64, path=K.PATHS["tc"]) == K.KDA_ERR_UNSUPPORTED


def test_decode_rejects_bad_args(K):
    d = K._lib.kda_decode_step
    assert d(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 96, 128, 128, 1, None) == K.KDA_ERR_INVALID_ARG
    assert d(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 96, 96, 128, 1, None) == K.KDA_ERR_UNSUPPORTED
    assert d(FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, 4, 96, 128, 128, 1, None) == K.KDA_ERR_INVALID_ARG
    assert d(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE + 8, FAKE, 4, 96, 128, 128, 1, None) == K.KDA_ERR_ALIGNMENT
    assert d(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 96, 128, 128, 3, None) == K.KDA_ERR_INVALID_ARG


REC = 74752  # bytes of one chunk's record: [-W ; Gamma q] + Gamma_C, Ut + P, Kh (73 KiB)


def al(x):
    return (x + 255) // 256 * 256


def test_workspace_and_launch_queries(K):
    # tensor-core shapes: the split form's per-chunk records
    assert K.kda_forward_workspace_size(1, 8192, 96, 128, 128, 64, 1, 1) == 128 * 96 * REC
    assert K.kda_forward_workspace_size(2, 8192, 96, 128, 128, 64, 2, 1) == 2 * 128 * 96 * REC
    assert K.kda_forward_workspace_size(2, 100, 3, 128, 128, 64, 2, 1) == 2 * 2 * 3 * REC
    # the pipe form: a ring of 4 records and 5 flags per unit
    assert K.kda_forward_workspace_size(2, 100, 3, 128, 128, 64, 2, 1, "tc_pipe") == \
        al(6 * 4 * REC) + al(6 * 5 * 4)
    assert K.kda_forward_workspace_size(2, 100, 3, 128, 128, 64, 2, 1, "tc_single") == 0
    # dense batches take the split form up to eight units per SM (1184 on 148 SMs), then the
    # single kernel (no workspace)
    assert K.kda_forward_workspace_size(12, 8192, 96, 128, 128, 64, 12, 1) == 12 * 128 * 96 * REC
    assert K.kda_forward_workspace_size(13, 8192, 96, 128, 128, 64, 13, 1) == 0
    assert K.kda_forward_launches(12, 8192, 96, 128, 128, 64, 1, 0, 12) == 2
    # packed sequences, up to three units per SM: records for at most T / 64 + N chunks per
    # head, the sequences' chunk offsets, and a small longest-first schedule (up to 2048)
    n_ch = -(-100000 // 64) + 3
    assert K.kda_forward_workspace_size(1, 100000, 96, 128, 128, 64, 3, 1) == \
        al(n_ch * 96 * REC) + al(4 * 4) + 256
    # more units than three per SM (8 x 96 = 768): AUTO runs the single form (its schedule only);
    # a forced split form still reports its records
    n_ch = -(-352549 // 64) + 8
    assert K.kda_forward_workspace_size(1, 352549, 96, 128, 128, 64, 8, 1) == 256
    assert K.kda_forward_workspace_size(1, 352549, 96, 128, 128, 64, 8, 1, "tc_split") == \
        al(n_ch * 96 * REC) + al(9 * 4) + 256
    with pytest.raises(K.KdaError):
        K.kda_forward_workspace_size(1, 352549, 96, 128, 128, 64, 8, 1, "tc_pipe")
    # other shapes (SIMT kernel): only the schedule
    assert K.kda_forward_workspace_size(1, 100000, 2, 64, 64, 32, 2048, 0) == 8192
    assert K.kda_forward_workspace_size(1, 100000, 2, 64, 64, 32, 2049, 0) == 0
    # launches: split = records + chains (+ chunk offsets and schedule for packed batches);
    # pipe = one launch, only for up to 197 units on 148 SMs
    assert K.kda_forward_launches(1, 352549, 96, 128, 128, 64, 1, 1, 8) == 2
    assert K.kda_forward_launches(1, 352549, 96, 128, 128, 64, 1, 1, 8, "tc_split") == 4
    assert K.kda_forward_launches(1, 100000, 96, 128, 128, 64, 1, 1, 3) == 4
    assert K.kda_forward_launches(1, 352549, 96, 128, 128, 64, 1, 1, 8, "tc_single") == 2
    assert K.kda_forward_launches(1, 352549, 96, 128, 128, 64, 1, 1, 8, "simt") == 2
    assert K.kda_forward_launches(1, 352549, 96, 128, 128, 64, 1, 1, 8, "tc_pipe") == -1
    assert K.kda_forward_launches(1, 8192, 96, 128, 128, 64, 1, 0, 1) == 2
    assert K.kda_forward_launches(1, 8192, 96, 128, 128, 64, 1, 0, 1, "tc_split") == 2
    assert K.kda_forward_launches(1, 8192, 96, 128, 128, 64, 1, 0, 1, "tc_pipe") == 1
    assert K.kda_forward_launches(1, 8192, 96, 128, 128, 64, 1, 0, 1, "tc_single") == 1
    assert K.kda_forward_launches(2, 8192, 99, 128, 128, 64, 1, 0, 2, "tc_pipe") == -1  # 198 units
    with pytest.raises(K.KdaError):
        K.kda_forward_workspace_size(1, 8192, 96, 100, 128, 64, 1, 1)
    assert K.kda_forward_launches(1, 256, 1, 32, 32, 16, 0, 0, 1, "simt") == 1
    assert K.kda_forward_launches(1, 256, 1, 48, 32, 16, 0, 0, 1) == -1
    # forcing a tensor-core form off its shapes is refused
    for f in ("tc_split", "tc_single", "tc_pipe"):
        assert K.kda_forward_launches(1, 256, 1, 32, 32, 16, 0, 0, 1, f) == -1


def test_python_binding_refuses_cpu_tensors(K):
    import torch
    x = torch.zeros(1, 4, 1, 32)
    with pytest.raises(ValueError, match="CUDA"):
        K.kda_forward(x, x, x, x, torch.zeros(1, 4, 1))


def seg(K, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, S0=None, o=FAKE, S_T=None, B=1, T=1000, H=2,
             dk=128, dv=128, chunk=64, dtype=1, seg_len=256, ws=None, ws_bytes=0, status=None, stream=None,
             path=0)
    a.update(kw)
    return K._lib.kda_forward_segmented(a["q"], a["k"], a["v"], a["g"], a["beta"], a["S0"], a["o"], a["S_T"],
                                        a["B"], a["T"], a["H"], a["dk"], a["dv"], a["chunk"], a["dtype"],
                                        a["seg_len"], a["ws"], a["ws_bytes"], a["status"], a["stream"],
                                        a["path"])


def test_segmented_rejects_bad_arguments(K):
    assert seg(K, seg_len=0) == K.KDA_ERR_INVALID_ARG
    assert seg(K, seg_len=100) == K.KDA_ERR_INVALID_ARG          # not a multiple of chunk
    assert seg(K, seg_len=-64) == K.KDA_ERR_INVALID_ARG
    assert seg(K, dk=48) == K.KDA_ERR_UNSUPPORTED
    assert seg(K, v=None) == K.KDA_ERR_INVALID_ARG
    assert seg(K, o=None) == K.KDA_ERR_INVALID_ARG
    assert seg(K, q=FAKE + 4) == K.KDA_ERR_ALIGNMENT
    # four segments need the workspace: missing or short -> rejected before launch
    assert seg(K) == K.KDA_ERR_WORKSPACE
    assert seg(K, ws=FAKE, ws_bytes=1024) == K.KDA_ERR_WORKSPACE
    # fp32 never takes the tensor-core kernel
    assert seg(K, dtype=0, path=K.PATHS["tc"]) == K.KDA_ERR_UNSUPPORTED


def test_segmented_queries(K):
    # 4 segments x 2 heads: three fp32 128 x 128 states per (segment, head), offsets, and on
    # the tensor-core shapes the records of every chunk of the segments (at most T / 64 + 4
    # chunks per head, 73 KiB each, with their own chunk offsets and schedule)
    n = K.kda_forward_segmented_workspace_size(1, 1000, 2, 128, 128, 64, 1, 256)
    states = 3 * 4 * 2 * 128 * 128 * 4
    records = al((-(-1000 // 64) + 4) * 2 * REC)
    assert n >= states + records and n < states + records + 4096
    # the transition of a dk = 64 segment is 64 x 64 whatever dv is
    n2 = K.kda_forward_segmented_workspace_size(1, 1000, 2, 64, 128, 64, 1, 256)
    assert n2 >= 4 * 2 * (64 * 64 + 2 * 128 * 64) * 4
    # one segment: the plain prefill's needs (the split form's records for a dense batch)
    assert K.kda_forward_segmented_workspace_size(2, 1000, 2, 128, 128, 64, 1, 1024) == 2 * 16 * 2 * REC
    assert K.kda_forward_segmented_launches(2, 1000, 2, 128, 128, 64, 1, 1024) == 2
    # tensor-core shapes: init, chunk offsets, schedule, records, three chain passes, scan
    assert K.kda_forward_segmented_launches(1, 1000, 2, 128, 128, 64, 1, 256) == 8
    # elsewhere: init, three prefill passes each with a longest-first schedule, scan
    assert K.kda_forward_segmented_launches(1, 1000, 2, 64, 64, 64, 1, 256) == 8
    with pytest.raises(K.KdaError):
        K.kda_forward_segmented_workspace_size(1, 1000, 2, 128, 128, 64, 1, 96)


def segv(K, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, S0=None, o=FAKE, S_T=None, T=1000, H=2,
             dk=128, dv=128, chunk=64, dtype=1, cu=FAKE, num=3, seg_len=256, ws=None, ws_bytes=0, status=None,
             stream=None, path=0)
    a.update(kw)
    return K._lib.kda_forward_segmented_varlen(a["q"], a["k"], a["v"], a["g"], a["beta"], a["S0"], a["o"],
                                               a["S_T"], a["T"], a["H"], a["dk"], a["dv"], a["chunk"], a["dtype"],
                                               a["cu"], a["num"], a["seg_len"], a["ws"], a["ws_bytes"],
                                               a["status"], a["stream"], a["path"])


def test_segmented_varlen_rejects_bad_arguments(K):
    assert segv(K, seg_len=0) == K.KDA_ERR_INVALID_ARG
    assert segv(K, seg_len=100) == K.KDA_ERR_INVALID_ARG
    assert segv(K, num=0) == K.KDA_ERR_INVALID_ARG
    assert segv(K, cu=None) == K.KDA_ERR_INVALID_ARG
    assert segv(K, dk=48) == K.KDA_ERR_UNSUPPORTED
    assert segv(K, o=None) == K.KDA_ERR_INVALID_ARG
    assert segv(K, k=FAKE + 4) == K.KDA_ERR_ALIGNMENT
    assert segv(K) == K.KDA_ERR_WORKSPACE
    assert segv(K, ws=FAKE, ws_bytes=4096) == K.KDA_ERR_WORKSPACE
    assert segv(K, dtype=0, path=K.PATHS["tc"]) == K.KDA_ERR_UNSUPPORTED


def test_segmented_varlen_queries(K):
    # T = 1000 over 3 sequences cut every 256 tokens: at most 1000 // 256 + 3 = 6 segments;
    # three fp32 states per (segment, head), and the records of every chunk (6 x 2 units)
    n = K.kda_forward_segmented_varlen_workspace_size(1000, 2, 128, 128, 64, 1, 3, 256)
    states = 3 * 6 * 2 * 128 * 128 * 4
    records = al((-(-1000 // 64) + 6) * 2 * REC)
    assert n >= states + records and n < states + records + 8192
    # segment plan, identity start, chunk offsets, schedule, records, three chain passes, scan
    assert K.kda_forward_segmented_varlen_launches(1000, 2, 128, 128, 64, 1, 3, 256) == 9
    # elsewhere: plan, identity start, three prefill passes each with a schedule, scan
    assert K.kda_forward_segmented_varlen_launches(1000, 2, 64, 64, 64, 1, 3, 256) == 9
    # more (segment, head) units than three per SM: single-kernel passes, no records
    big = K.kda_forward_segmented_varlen_workspace_size(100000, 96, 128, 128, 64, 1, 8, 4096)
    assert big < 3 * (100000 // 4096 + 8) * 96 * 128 * 128 * 4 + (1 << 20)
    # T <= seg_len: no sequence is cut, the plain packed prefill's needs
    assert K.kda_forward_segmented_varlen_workspace_size(1000, 2, 128, 128, 64, 1, 3, 1024) == \
        K.kda_forward_workspace_size(1, 1000, 2, 128, 128, 64, 3, 1)
    assert K.kda_forward_segmented_varlen_launches(1000, 2, 128, 128, 64, 1, 3, 1024, "auto") == \
        K.kda_forward_launches(1, 1000, 2, 128, 128, 64, 1, 1, 3)
    with pytest.raises(K.KdaError):
        K.kda_forward_segmented_varlen_workspace_size(1000, 2, 128, 128, 64, 1, 3, 96)


def test_decode_multi_rejects_bad_args(K):
    d = K._lib.kda_decode_multi
    args = lambda **kw: [kw.get(n, FAKE) for n in ("q", "k", "v", "g", "beta", "S", "o", "acc")] + \
        [kw.get(n, x) for n, x in (("N", 4), ("T", 3), ("H", 2), ("dk", 128), ("dv", 128), ("dt", 1))] + \
        [kw.get("status"), None]
    assert d(*args(T=0)) == K.KDA_ERR_INVALID_ARG
    assert d(*args(N=0)) == K.KDA_ERR_INVALID_ARG
    assert d(*args(T=65)) == K.KDA_ERR_UNSUPPORTED
    assert d(*args(dk=96)) == K.KDA_ERR_UNSUPPORTED
    assert d(*args(S=None)) == K.KDA_ERR_INVALID_ARG
    assert d(*args(S=FAKE + 8)) == K.KDA_ERR_ALIGNMENT
    assert d(*args(acc=FAKE + 4)) == K.KDA_ERR_ALIGNMENT
    assert d(*args(dt=5)) == K.KDA_ERR_INVALID_ARG
    assert d(*args(status=FAKE + 4)) == K.KDA_ERR_ALIGNMENT


def test_snapshots_reject_bad_arguments(K):
    f = K._lib.kda_forward_snapshots
    base = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, S0=None, o=FAKE, S_T=None, snap=FAKE, every=256,
                B=1, T=1000, H=2, dk=128, dv=128, chunk=64, dt=1, ws=None, wsb=0, st=None, stream=None, path=0)
    call = lambda **kw: f(*[dict(base, **kw)[n] for n in base])
    assert call(every=0) == K.KDA_ERR_INVALID_ARG
    assert call(every=100) == K.KDA_ERR_INVALID_ARG     # not a multiple of chunk
    assert call(snap=None) == K.KDA_ERR_INVALID_ARG     # 3 snapshots are due
    assert call(snap=FAKE + 4) == K.KDA_ERR_ALIGNMENT
    assert call(dk=48) == K.KDA_ERR_UNSUPPORTED
    # the pipe form writes no snapshots; the split form stores them for up to one unit per SM
    assert call(path=K.PATHS["tc_pipe"]) == K.KDA_ERR_UNSUPPORTED
    assert call(path=K.PATHS["tc_split"], B=2, H=75) == K.KDA_ERR_UNSUPPORTED
    # a forced split form needs its records
    assert call(path=K.PATHS["tc_split"]) == K.KDA_ERR_WORKSPACE


def test_pair_and_scan_reject_bad_arguments(K):
    pair = K._lib.kda_segment_pair
    assert pair(FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, 1, 64, 2, 128, 128, 64, 1, None, None, 0) == K.KDA_ERR_INVALID_ARG
    assert pair(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE + 4, FAKE, 1, 64, 2, 128, 128, 64, 1, None, None, 0) == K.KDA_ERR_ALIGNMENT
    assert pair(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 64, 2, 48, 128, 64, 1, None, None, 0) == K.KDA_ERR_UNSUPPORTED
    scan = K._lib.kda_kcp_scan
    assert scan(None, FAKE, FAKE, FAKE, None, 1, 0, 2, 128, 128, None) == K.KDA_ERR_INVALID_ARG
    assert scan(None, None, FAKE, FAKE, None, 1, 2, 2, 128, 128, None) == K.KDA_ERR_INVALID_ARG
    assert scan(None, FAKE, FAKE, FAKE, None, 1, 2, 2, 96, 128, None) == K.KDA_ERR_UNSUPPORTED
    assert scan(FAKE + 8, FAKE, FAKE, FAKE, None, 1, 2, 2, 128, 128, None) == K.KDA_ERR_ALIGNMENT


def test_fused_entry_points_reject_unknown_flags(K):
    f = K._lib.kda_forward_fused
    base = [FAKE] * 5 + [None, FAKE, None, 1, 64, 2, 128, 128, 64, 1, None, 0, None, 0, None, None, 0]
    assert f(*base, 4) == K.KDA_ERR_INVALID_ARG
    assert f(*(base[:8] + [0] + base[9:]), 1) == K.KDA_ERR_INVALID_ARG  # B = 0
    # the pipe form has no fused variant; a forced split form needs its records
    assert f(*(base[:-1] + [K.PATHS["tc_pipe"]]), 1) == K.KDA_ERR_UNSUPPORTED
    assert f(*(base[:-1] + [K.PATHS["tc_split"]]), 1) == K.KDA_ERR_WORKSPACE
    d = K._lib.kda_decode_step_fused
    assert d(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 96, 128, 128, 1, None, 8) == K.KDA_ERR_INVALID_ARG


def test_host_entry_point_validates_before_any_cuda_call(K):
    f = K._lib.kda_forward_host

    def call(**kw):
        a = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, S0=None, o=FAKE, S_T=None, B=1, T=256, H=2,
                 dk=128, dv=128, chunk=64, dtype=1, piece=128, ws=FAKE, ws_bytes=1 << 40, status=None,
                 stream=None, path=0)
        a.update(kw)
        return f(a["q"], a["k"], a["v"], a["g"], a["beta"], a["S0"], a["o"], a["S_T"], a["B"], a["T"], a["H"],
                 a["dk"], a["dv"], a["chunk"], a["dtype"], a["piece"], a["ws"], a["ws_bytes"], a["status"],
                 a["stream"], a["path"])

    assert call(piece=100) == K.KDA_ERR_INVALID_ARG      # not whole chunks
    assert call(piece=-64) == K.KDA_ERR_INVALID_ARG
    assert call(dk=48) == K.KDA_ERR_UNSUPPORTED
    assert call(B=0) == K.KDA_ERR_INVALID_ARG
    assert call(dtype=0, path=K.PATHS["tc"]) == K.KDA_ERR_UNSUPPORTED
    for name in ("q", "k", "v", "g", "beta", "o"):
        assert call(**{name: None}) == K.KDA_ERR_INVALID_ARG, name
    assert call(ws=None) == K.KDA_ERR_WORKSPACE
    assert call(ws_bytes=1024) == K.KDA_ERR_WORKSPACE
    assert call(ws=FAKE + 16) == K.KDA_ERR_ALIGNMENT    # device workspace: 256-byte aligned


def test_host_workspace_size_is_two_piece_slots_and_the_state(K):
    # two slots of one piece's q, k, v, g, beta and o (each rounded up to 256 bytes), the fp32
    # state, and the device prefill's workspace for one piece (the split form's records)
    B, T, H, d, L = 1, 8192, 96, 128, 1024
    piece = B * L * H * d * 2
    slot = 5 * piece + B * L * H * 2
    state = B * H * d * d * 4
    records = K.kda_forward_workspace_size(B, L, H, d, d, 64, B, 1)
    assert records == B * (L // 64) * H * REC
    assert K.kda_forward_host_workspace_size(B, T, H, d, d, 64, 1, L) == 2 * slot + state + records
    # piece_len 0: about T / 8 in whole chunks; a piece never exceeds the sequence
    assert K.kda_forward_host_workspace_size(B, T, H, d, d, 64, 1, 0) == 2 * slot + state + records
    small = K.kda_forward_host_workspace_size(2, 100, 3, 64, 32, 32, 0, 256)
    tok = 2 * 100 * 3
    rnd = lambda x: (x + 255) // 256 * 256
    assert small == 2 * (3 * rnd(tok * 64 * 4) + 2 * rnd(tok * 32 * 4) + rnd(tok * 4)) + rnd(2 * 3 * 32 * 64 * 4)
    with pytest.raises(K.KdaError):
        K.kda_forward_host_workspace_size(1, 64, 2, 128, 128, 64, 1, 96)


def test_host_varlen_validates_offsets_before_any_cuda_call(K):
    import ctypes
    f = K._lib.kda_forward_host_varlen

    def call(cu, T=1000, num=None, **kw):
        arr = (ctypes.c_int32 * len(cu))(*cu)
        a = dict(ws=FAKE, ws_bytes=1 << 40, piece=256, path=0)
        a.update(kw)
        return f(FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, None, T, 2, 128, 128, 64, 1, arr,
                 len(cu) - 1 if num is None else num, a["piece"], a["ws"], a["ws_bytes"], None, None, a["path"])
    assert call([1, 500, 1000]) == K.KDA_ERR_INVALID_ARG       # does not start at 0
    assert call([0, 600, 500, 1000]) == K.KDA_ERR_INVALID_ARG  # decreasing
    assert call([0, 500, 999]) == K.KDA_ERR_INVALID_ARG        # does not end at T
    assert call([0, 1000], num=0) == K.KDA_ERR_INVALID_ARG
    assert call([0, 500, 1000], piece=100) == K.KDA_ERR_INVALID_ARG  # not whole chunks
    assert call([0, 500, 1000], ws=None) == K.KDA_ERR_WORKSPACE
    assert call([0, 500, 1000], ws=FAKE + 16) == K.KDA_ERR_ALIGNMENT
    # the workspace: two slots of the largest piece, every sequence's state, the pieces'
    # offsets, the device prefill's scratch for the largest piece
    n2 = K.kda_forward_host_varlen_workspace_size(1000, 2, 128, 128, 64, 1, [0, 500, 1000], 256)
    n8 = K.kda_forward_host_varlen_workspace_size(1000, 2, 128, 128, 64, 1, [0] + [125 * i for i in range(1, 9)], 256)
    assert n2 > 2 * 256 * 2 * 128 * 2 * 5 and n8 > n2
    with pytest.raises(K.KdaError):
        K.kda_forward_host_varlen_workspace_size(1000, 2, 128, 128, 64, 1, [0, 500, 900], 256)
