"""A line-by-line Python model of the decode kernel's schedule (decode_kernel.cuh): the stream-K
split of all KV blocks over the worker warps, each warp's windows of 32 block ids, its copy ring of
NS stages, its segments and the partial slots and tickets of split (sequence, head group) units.

Run on random batches (empty and one-block sequences, lengths clamped by max_context_len and the
table width, worker counts from 1 to a full B200), it checks what the kernel relies on:
  - every block of every unit is computed exactly once, and units with no blocks get zero output;
  - a warp never waits on a ring stage it has not issued, and reuses a stage only after the block
    issued NS positions earlier has been computed;
  - a unit split between warps is covered by contiguous segments of consecutive warps, exactly the
    warps w_first..w_last that the ticket counts, and their partial slots u + w are unique and
    inside the workspace (U + W slots).
The model carries no arithmetic; the CUDA kernel's results are checked against the oracle by the
GPU parity tests.
"""
import random

import pytest


def clamp_len(L, max_ctx, mbps, BS): return max(0, min(L, min(max_ctx, mbps*BS)))
def owner_of(g, T, W): return ((g+1)*W - 1)//T

def simulate(lens, HG, BS, NS, W, max_ctx, mbps):
    S=len(lens)
    Lc=[clamp_len(L,max_ctx,mbps,BS) for L in lens]
    nblk=[(L+BS-1)//BS for L in Lc]
    T=HG*sum(nblk)
    consumed={}
    seg_records={}  # unit -> list of (w, j0, j1)
    zeroed=set()
    U=S*HG
    for w in range(W):
        for s in range(S):
            if Lc[s]==0:
                for hg in range(HG):
                    if (s*HG+hg)%W==w: zeroed.add((s,hg))
        if T==0: continue
        We=min(W,T)
        if w>=We: continue
        start=w*T//We; end=(w+1)*T//We
        assert start<end
        # locate
        acc=0; s0=None
        for s in range(S):
            cnt=nblk[s]*HG
            if acc+cnt>start: s0=s; seq_p0=acc; break
            acc+=cnt
        assert s0 is not None
        o=start-seq_p0; hg=o//nblk[s0]; j0=o%nblk[s0]
        cur=dict(s=s0,hg=hg,j0=j0,L=Lc[s0],nblk=nblk[s0],p0=start,seq_p0=seq_p0)
        cur['n']=min(min(32,cur['nblk']-cur['j0']), end-start)
        def next_win(a):
            b=dict(a); b['p0']=a['p0']+a['n']; b['n']=0
            if a['n']==0 or b['p0']>=end: return b
            b['j0']=a['j0']+a['n']
            if b['j0']>=a['nblk']:
                b['j0']=0; b['hg']=a['hg']+1
                if b['hg']>=HG:
                    b['hg']=0; b['seq_p0']=a['seq_p0']+HG*a['nblk']
                    s=a['s']; L=0
                    while True:
                        s+=1; L=Lc[s] if s<S else 0
                        if not (L==0 and s<S): break
                    b['s']=s; b['L']=L; b['nblk']=(L+BS-1)//BS
            b['n']=min(min(32,b['nblk']-b['j0']), end-b['p0'])
            return b
        nxt=next_win(cur)
        issued=set(); pos=start; iss=start; seg_j0=cur['j0']
        def win_of(x):
            if x < cur['p0']+cur['n']: return cur
            if nxt['n']>0 and x < nxt['p0']+nxt['n']: return nxt
            return None
        while pos<end:
            if pos==cur['p0']+cur['n']:
                new_unit=(nxt['s']!=cur['s']) or (nxt['hg']!=cur['hg'])
                cur=nxt; nxt=next_win(cur)
                assert cur['n']>0
                if new_unit: seg_j0=cur['j0']
            lim=min(pos+NS,end)
            while iss<lim:
                wi=win_of(iss)
                if wi is None: break
                k=iss-wi['p0']; assert 0<=k<32
                j=wi['j0']+k; assert j<wi['nblk'] and j<mbps
                # stage reuse: position iss-NS must be consumed already
                assert iss-NS < pos
                issued.add(iss); iss+=1
            assert pos in issued, "waiting on a position never issued"
            kw=pos-cur['p0']; assert 0<=kw<cur['n']
            j=cur['j0']+kw
            key=(cur['s'],cur['hg'],j)
            assert key not in consumed; consumed[key]=w
            # position check
            assert pos == cur['seq_p0'] + cur['hg']*cur['nblk'] + j
            pos+=1
            j_end=j+1
            if j_end==cur['nblk'] or pos==end:
                u=cur['s']*HG+cur['hg']
                seg_records.setdefault(u,[]).append((w,seg_j0,j_end, cur['seq_p0']+cur['hg']*cur['nblk']))
                seg_j0=j_end
    # every (s, hg, j) consumed exactly once
    for s in range(S):
        for hg in range(HG):
            for j in range(nblk[s]):
                assert (s,hg,j) in consumed, (s,hg,j)
            if nblk[s]==0: assert (s,hg) in zeroed
    assert len(consumed)==T
    # segments: cover each unit contiguously; n_seg formula; slots in range and unique
    slots=set()
    for u,segs in seg_records.items():
        segs.sort(key=lambda x:x[1])
        s,hg=divmod(u,HG)
        assert segs[0][1]==0 and segs[-1][2]==nblk[s]
        for a,b in zip(segs,segs[1:]): assert a[2]==b[1]
        unit_p0=segs[0][3]
        We=min(W,T)
        wf=owner_of(unit_p0,T,We); wl=owner_of(unit_p0+nblk[s]-1,T,We)
        ws=[x[0] for x in segs]
        if len(segs)>1 or segs[0][1]!=0 or segs[0][2]!=nblk[s]:
            assert ws==list(range(wf,wl+1)), (ws,wf,wl)
            for ww in ws:
                sl=u+ww; assert 0<=sl<U+W; assert sl not in slots; slots.add(sl)
        else:
            assert wf==wl==ws[0]
    return T


@pytest.mark.parametrize("seed", range(4))
def test_schedule_model_random_batches(seed):
    rng = random.Random(seed)
    for _ in range(400):
        BS = rng.choice([16, 32])
        HG = rng.choice([1, 2, 4, 8, 32])
        NS = rng.choice([2, 3, 4, 6])
        S = rng.randint(1, 40)
        lens = [rng.choice([0, 1, 2, 15, 16, 17, 31, 32, 33, rng.randint(0, 3000)]) for _ in range(S)]
        max_ctx = max(lens) if rng.random() < 0.8 else rng.randint(0, 3000)
        mbps = max(1, (max(lens) + BS - 1) // BS) if rng.random() < 0.8 else rng.randint(1, 100)
        W = rng.choice([1, 4, 8, 32, 100, 592, 1776, 2368])
        simulate(lens, HG, BS, NS, W, max_ctx, mbps)
