"""The C ABI without a GPU: the library loads, exports every function include/tr.h declares,
computes the tail length exactly, and rejects bad arguments before touching the device."""
import ctypes
import os
import random
import re

import pytest

import oracle
import linear_attention_state_zero_b200 as tr

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = 0x10000  # a 16-byte aligned non-NULL address; never dereferenced by validation


def header_functions():
    src = open(os.path.join(ROOT, "include", "tr.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tr_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_function_is_exported():
    names = header_functions()
    assert len(names) >= 14
    for n in names:
        assert hasattr(tr.lib, n), n
        assert n in tr._SIGNATURES, "binding lacks a signature for " + n


def test_struct_layouts_match_c():
    # offsets follow the C declaration order with natural alignment
    assert ctypes.sizeof(tr.ScanArgs) == 16 + 8 + 12 + 4 + 24 + 8 * 10
    assert tr.ScanArgs.q_stride.offset == 40
    assert ctypes.sizeof(tr.LALayer) == 88
    assert tr.LALayer.W_down.offset == 48 and tr.LALayer.o_norm_gain.offset == 80
    assert tr.GroupArgs.d_ff.offset == 44
    assert tr.GroupArgs.h_tail.offset == 48
    assert tr.GroupArgs.conv_width.offset == 96 and tr.GroupArgs.conv_state.offset == 104
    assert ctypes.sizeof(tr.GroupArgs) == 112


def test_tail_len_matches_oracle():
    r = random.Random(5)
    for _ in range(2000):
        m = r.randint(0, 1 << 20)
        num = r.randint(0, 120)
        den = r.choice([1, 10, 100, 1000, 7])
        assert tr.tail_len(m, num, den) == oracle.tail_len(m, num, den)
    assert tr.tail_len(10000, 5, 100) == 500
    assert tr.tail_len(100, 7, 100) == 7
    assert tr.lib.tr_tail_len(10, 1, 0) == -1
    assert tr.lib.tr_tail_len(-1, 1, 2) == -1


def _scan_args(**kw):
    cu = (ctypes.c_int32 * 3)(0, 5, 9)
    a = tr.ScanArgs(2, 4, 128, 128, 9, tr.TR_DTYPE_BF16, 0, 1.0, 0, 0, 0,
                    FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ctypes.addressof(cu), None, FAKE, FAKE + 4096)
    for k, v in kw.items():
        setattr(a, k, v)
    return a, cu


@pytest.mark.parametrize("field,value,status", [
    ("n_heads", 0, 1), ("dtype", 7, 3), ("d_k", 96, 5), ("d_v", 32, 5), ("flags", 0x80, 1),
    ("k", None, 1), ("S_final", None, 1), ("cu_seqlens", None, 1), ("total_tokens", 10, 2), ("q", FAKE + 2, 4),
    ("k_stride", 100, 2), ("S0", FAKE + 4096, 1), ("cu_seqlens_host", None, 1),
])
def test_scan_rejects_bad_arguments(field, value, status):
    a, cu = _scan_args(**{field: value})
    st = tr.lib.tr_gdn_scan(ctypes.byref(a), None, 0, None)
    assert st == status, (st, tr.lib.tr_last_error())
    assert tr.lib.tr_last_error()


def test_transition_product_checks():
    """tr_transition_product sizes its workspace (the zero v and the identities, then the
    scan's) and rejects bad arguments before any device work."""
    a, cu = _scan_args()
    need = tr.lib.tr_transition_product_workspace_size(ctypes.byref(a))
    T, H, d, N = 9, 4, 128, 2
    assert need >= T * H * d * 2 + N * H * d * d * 4
    tp = tr.lib.tr_transition_product
    assert tp(ctypes.byref(a), None, FAKE, need, None) == 1          # P NULL
    assert tp(ctypes.byref(a), FAKE + 4, FAKE, need, None) == 4      # P misaligned
    assert tp(ctypes.byref(a), FAKE, None, need, None) == 6          # no workspace
    assert tp(ctypes.byref(a), FAKE, FAKE, need - 1, None) == 6      # too small
    assert tp(ctypes.byref(a), FAKE, FAKE + 16, need, None) == 4     # not 256-byte aligned
    b, cu_b = _scan_args(d_k=96)
    assert tr.lib.tr_transition_product_workspace_size(ctypes.byref(b)) == 0
    assert tp(ctypes.byref(b), FAKE, FAKE, 1 << 30, None) == 5


def test_scan_rejects_bad_cu_seqlens():
    a, _ = _scan_args()
    bad = (ctypes.c_int32 * 3)(0, 6, 5)
    a.cu_seqlens_host = ctypes.addressof(bad)
    assert tr.lib.tr_gdn_scan(ctypes.byref(a), None, 0, None) == 2


def _group_args(**kw):
    cu = (ctypes.c_int32 * 2)(0, 16)
    layers = (tr.LALayer * 3)(*[tr.LALayer(None, FAKE, FAKE) for _ in range(3)])
    a = tr.GroupArgs(1, 16, 128, 128, 2048, 3, 16, 0, 0.0, 0.0, 0, FAKE, FAKE,
                     ctypes.addressof(cu), layers, FAKE, None)
    for k, v in kw.items():
        setattr(a, k, v)
    return a, (cu, layers)


@pytest.mark.parametrize("field,value,status", [
    ("n_layers", 0, 5), ("n_layers", 65, 5), ("d_model", 100, 5), ("d_k", 32, 5),
    ("flags", 32, 1), ("d_ff", 100, 5), ("conv_width", 5, 5), ("conv_width", 1, 5),
    ("conv_width", 4, 1), ("conv_state", FAKE, 1), ("d_ff", -128, 5), ("h_tail", None, 1), ("S_hat", FAKE + 8, 4), ("total_tokens", 17, 2),
])
def test_replay_rejects_bad_arguments(field, value, status):
    a, keep = _group_args(**{field: value})
    assert tr.lib.tr_replay_group(ctypes.byref(a), None, 0, None) == status


def test_replay_skip_flag_forbids_x_out():
    a, keep = _group_args(flags=tr.TR_SKIP_LAST_OUTPUT, x_out=FAKE)
    assert tr.lib.tr_replay_group(ctypes.byref(a), None, 0, None) == 1


@pytest.mark.parametrize("ffn,d_ff,status", [   # ffn = (ffn_gain, W_gate, W_up, W_down)
    ((None, None, FAKE, FAKE), 256, 1),         # W_gate NULL but W_up/W_down given
    ((None, FAKE, None, FAKE), 256, 1),         # W_up NULL
    ((None, FAKE, FAKE, None), 256, 1),         # W_down NULL
    ((None, FAKE, FAKE, FAKE + 8), 256, 4),     # misaligned W_down
    ((FAKE + 4, FAKE, FAKE, FAKE), 256, 4),     # misaligned ffn_gain
    ((None, FAKE, FAKE, FAKE), 0, 1),           # FFN weights with d_ff = 0
])
def test_replay_rejects_bad_ffn(ffn, d_ff, status):
    a, keep = _group_args(d_ff=d_ff)
    lw = keep[1][1]
    lw.ffn_gain, lw.W_gate, lw.W_up, lw.W_down = ffn
    assert tr.lib.tr_replay_group(ctypes.byref(a), None, 0, None) == status, \
        tr.lib.tr_last_error()


def test_replay_ffn_workspace_and_kernel_count():
    """The FFN's hidden activation [T, d_ff] bf16 is in the workspace; each FFN that runs adds
    three kernels, and the tail-FFN skip drops the last one."""
    a, keep = _group_args()
    base_ws = tr.lib.tr_replay_group_workspace_size(ctypes.byref(a))
    base_n = tr.lib.tr_replay_group_kernel_count(ctypes.byref(a))
    a.d_ff = 1024
    for lw in keep[1]:
        lw.W_gate, lw.W_up, lw.W_down = FAKE, FAKE, FAKE
    assert tr.lib.tr_replay_group_workspace_size(ctypes.byref(a)) >= base_ws + 16 * 1024 * 2
    # x_out NULL: the last layer's output (and so its FFN) is not computed
    assert tr.lib.tr_replay_group_kernel_count(ctypes.byref(a)) == base_n + 2 * 3
    a.x_out = FAKE + 4096
    with_out = tr.lib.tr_replay_group_kernel_count(ctypes.byref(a))
    a.flags = tr.TR_SKIP_LAST_FFN
    assert with_out == tr.lib.tr_replay_group_kernel_count(ctypes.byref(a)) + 3


def test_replay_rejects_bad_gdn_options():
    # d_k != d_v with the convolution
    a, keep = _group_args(conv_width=4, d_v=64)
    for lw in keep[1]:
        lw.conv_w = FAKE
    assert tr.lib.tr_replay_group(ctypes.byref(a), None, 0, None) == 5
    # conv_w on a layer without conv_width
    a, keep = _group_args()
    keep[1][2].conv_w = FAKE
    assert tr.lib.tr_replay_group(ctypes.byref(a), None, 0, None) == 1
    # o_norm_gain without the output gate; misaligned gate parameters
    a, keep = _group_args()
    keep[1][0].o_norm_gain = FAKE
    assert tr.lib.tr_replay_group(ctypes.byref(a), None, 0, None) == 1
    a, keep = _group_args()
    keep[1][1].A_log = FAKE + 2
    assert tr.lib.tr_replay_group(ctypes.byref(a), None, 0, None) == 4
    # misaligned convolution state
    a, keep = _group_args(conv_width=4, conv_state=FAKE + 8)
    for lw in keep[1]:
        lw.conv_w = FAKE
    assert tr.lib.tr_replay_group(ctypes.byref(a), None, 0, None) == 4


def test_replay_gdn_workspace_and_kernel_count():
    """The convolution adds one kernel per layer and a [T, 2Hd_k + Hd_v] bf16 buffer; the output
    gate adds one kernel per computed output and a [T, H d_v] bf16 buffer."""
    a, keep = _group_args()
    ws0 = tr.lib.tr_replay_group_workspace_size(ctypes.byref(a))
    n0 = tr.lib.tr_replay_group_kernel_count(ctypes.byref(a))
    T, H, d = 16, 16, 128
    a.conv_width = 4
    for lw in keep[1]:
        lw.conv_w = FAKE
    assert tr.lib.tr_replay_group_kernel_count(ctypes.byref(a)) == n0 + 3
    assert tr.lib.tr_replay_group_workspace_size(ctypes.byref(a)) >= ws0 + T * 3 * H * d * 2
    a.flags = tr.TR_OUTPUT_GATE
    # x_out NULL: outputs of layers 0 and 1 only
    assert tr.lib.tr_replay_group_kernel_count(ctypes.byref(a)) == n0 + 3 + 2
    assert tr.lib.tr_replay_group_workspace_size(ctypes.byref(a)) >= ws0 + T * 4 * H * d * 2


def test_overlapped_replay_checks_everything_before_the_copy():
    """tr_replay_groups_overlapped rejects its KV arguments and every group argument before
    it issues the copy (a rejected call moves no bytes and needs no device)."""
    a, keep = _group_args()
    arr = (tr.GroupArgs * 1)(a)
    need = tr.lib.tr_replay_groups_workspace_size(arr, 1)
    ov = tr.lib.tr_replay_groups_overlapped
    S1, S2 = FAKE, FAKE + 64          # two distinct stream handles (never used)
    assert ov(arr, 1, FAKE, need, FAKE, FAKE, 4096, S1, S1) == 1      # one stream for both
    assert ov(arr, 1, FAKE, need, None, FAKE, 4096, S1, S2) == 1      # KV source NULL
    assert ov(arr, 1, FAKE, need - 1, FAKE, FAKE, 4096, S1, S2) == 6  # workspace too small
    bad = (tr.GroupArgs * 2)(a, a)
    bad[1].n_layers = 0
    assert ov(bad, 2, FAKE, need, FAKE, FAKE, 4096, S1, S2) == 5      # group 1 invalid
    assert "group 1" in tr.lib.tr_last_error().decode()
    assert ov(arr, -1, FAKE, need, FAKE, FAKE, 4096, S1, S2) == 1


def test_lanes_workspace_is_whole_slices():
    """tr_replay_groups' lanes: L slices of the single-group workspace (256-byte multiples),
    1 <= L <= 4; anything else is 0."""
    a, keep = _group_args()
    arr = (tr.GroupArgs * 2)(a, a)
    one = tr.lib.tr_replay_groups_workspace_size(arr, 2)
    assert one > 0 and one % 256 == 0
    for lanes in range(1, 5):
        assert tr.lib.tr_replay_groups_lanes_workspace_size(arr, 2, lanes) == lanes * one
    assert tr.lib.tr_replay_groups_lanes_workspace_size(arr, 2, 0) == 0
    assert tr.lib.tr_replay_groups_lanes_workspace_size(arr, 2, 5) == 0


def test_replay_workspace_checks():
    a, keep = _group_args()
    need = tr.lib.tr_replay_group_workspace_size(ctypes.byref(a))
    T, D, H, d = 16, 2048, 16, 128
    assert need >= T * D * 4 + T * D * 2 + T * (3 * H * d) * 2 + T * H * d * 2
    assert tr.lib.tr_replay_group(ctypes.byref(a), None, 0, None) == 6
    assert tr.lib.tr_replay_group(ctypes.byref(a), FAKE, need - 1, None) == 6
    assert tr.lib.tr_replay_group(ctypes.byref(a), FAKE + 16, need, None) == 4


def test_state_error_workspace_and_args():
    assert tr.lib.tr_state_error_workspace_size(0) == 0
    assert tr.lib.tr_state_error_workspace_size(100) >= 1600
    assert tr.lib.tr_state_error(FAKE, FAKE, 100, 128, 128, FAKE, FAKE, None, 0, None) == 6
    assert tr.lib.tr_state_error(FAKE, FAKE + 4, 1, 8, 8, None, FAKE, FAKE, 4096, None) == 4
    assert tr.lib.tr_state_error(FAKE, FAKE, -1, 8, 8, None, FAKE, FAKE, 4096, None) == 1


def test_replay_kernel_names_match_the_count():
    """tr_replay_group_kernel_names lists exactly the launches tr_replay_group_kernel_count
    counts, in launch order: the first layer's RMSNorm (later layers' is folded into the
    residual GEMM before them), per layer the input projection, the scan's kernels and the
    output projection (not after the last layer without x_out), plus the options'."""
    a, keep = _group_args()
    names = tr.lib.tr_replay_group_kernel_names(ctypes.byref(a)).decode().split(",")
    assert len(names) == tr.lib.tr_replay_group_kernel_count(ctypes.byref(a))
    assert names[:2] == ["rmsnorm", "in_proj"] and names[-1] != "out_proj"
    assert names.count("rmsnorm") == 1 and names.count("out_proj") == 2
    assert all(n.startswith("scan") for n in names if n not in ("rmsnorm", "in_proj", "out_proj"))
    a.d_ff = 1024
    a.conv_width = 4
    a.flags = tr.TR_OUTPUT_GATE
    for lw in keep[1]:
        lw.W_gate, lw.W_up, lw.W_down, lw.conv_w = FAKE, FAKE, FAKE, FAKE
    names = tr.lib.tr_replay_group_kernel_names(ctypes.byref(a)).decode().split(",")
    assert len(names) == tr.lib.tr_replay_group_kernel_count(ctypes.byref(a))
    assert names.count("short_conv") == 3 and names.count("gated_norm") == 2
    assert names.count("ffn_gate_up") == 2 and names.count("ffn_down") == 2
    assert tr.lib.tr_replay_group_kernel_names(None) == b""


def test_wait_limit_setting_is_host_only_and_checked():
    """tr_set_wait_limit_ns accepts up to 60 s (0 = the default) and rejects more; it only
    sets a host value that later scan launches carry."""
    assert tr.lib.tr_set_wait_limit_ns(61_000_000_000) == 1
    assert tr.lib.tr_set_wait_limit_ns(1_000_000) == 0
    assert tr.lib.tr_set_wait_limit_ns(0) == 0
