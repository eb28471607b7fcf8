"""libsala: SALA hybrid sparse + linear attention prefill/decode on B200 (sm_100a)."""
