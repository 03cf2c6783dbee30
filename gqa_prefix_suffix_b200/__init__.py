"""B200 (sm_100a) suffix attention of the DM0.5 action expert."""
