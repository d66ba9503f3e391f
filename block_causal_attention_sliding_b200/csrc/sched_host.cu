// sched_host.cu -- inspection hook for the full-path schedules: enumerates on the host the
// pieces that every CTA (or CTA pair) of the persistent, three-buffer and CTA-pair kernels
// processes, with the same schedule code the kernels run.  Host only; used by the tests to check
// that every (unit, key tile) is covered exactly once and that split pieces merge as the kernels
// expect.
#include "persist_sched.cuh"
#include "tri_common.cuh"

extern "C" int sw_attn_schedule_pieces(int schedule, int nqt, int nt, int bh, int ctas, int32_t* out, int cap) {
    if (!out || cap < 0 || nqt < 1 || nt < 1 || bh < 1 || ctas < 1) return SW_EINVAL;
    if (schedule != SW_SCHED_PERSISTENT && schedule != SW_SCHED_TRI && schedule != SW_SCHED_PAIR) return SW_EINVAL;
    int n = 0;
    auto put = [&](int g, int unit, int j0, int j1, bool sk, int live) -> bool {
        if (n >= cap) return false;
        int32_t* r = out + 6 * (size_t)n;
        r[0] = g; r[1] = unit; r[2] = j0; r[3] = j1; r[4] = sk ? 1 : 0; r[5] = live;
        ++n;
        return true;
    };
    for (int g = 0; g < ctas; ++g) {
        if (schedule == SW_SCHED_PERSISTENT) {
            swattn::Sched s;
            s.init(nqt, nt, bh, ctas, g);
            swattn::PieceIt it;
            swattn::Piece pc;
            while (swattn::next_piece(s, it, pc))
                if (!put(g, pc.bh * s.npairs + pc.pair, pc.j0, pc.j1, pc.sk, pc.live)) return SW_ESHAPE;
        } else {
            // three-buffer kernel: units are Q tiles; CTA-pair kernel: units are pairs of Q tiles
            // (the second may not exist) over `ctas` clusters
            const int units = schedule == SW_SCHED_PAIR ? (nqt + 1) / 2 : nqt;
            swattn::tri::Sched s;
            s.init(units, nt, bh, ctas, g);
            swattn::tri::PieceIt it;
            swattn::tri::Piece pc;
            while (swattn::tri::next_piece(s, it, pc)) {
                const int live = schedule == SW_SCHED_PAIR ? (2 * (pc.unit % units) + 1 < nqt ? 2 : 1) : 1;
                if (!put(g, pc.unit, pc.j0, pc.j1, pc.sk, live)) return SW_ESHAPE;
            }
        }
    }
    return n;
}
