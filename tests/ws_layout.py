"""The forward workspace's size for a launch plan, written out from the
layout the public header documents, for tests that check the planner."""


def ws_bytes(batch, chunks, d_inner):
    """Forward workspace for a plan of `chunks` time chunks: a 256-byte status
    header, then per carried chunk boundary and sequence the writer tags (one
    u64 per channel octet), the end states (16 fp32 per channel) and the
    step-size sums (one fp32 per channel), each region 256-byte aligned."""
    def a(b):
        return (b + 255) // 256 * 256

    c = chunks - 1
    return 256 + a(c * batch * d_inner // 8 * 8) + a(c * batch * 16 * d_inner * 4) + a(c * batch * d_inner * 4)
