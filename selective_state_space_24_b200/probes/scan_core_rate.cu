// scan_core_rate.cu -- register-only model of one S6 step (two channels x 16
// states per thread: v = dt A, e = 2^v, h = e h + dt x B, y += C h), with and
// without the per-step softplus / SiLU transcendentals, at several CTAs per
// SM.  It bounds what the full kernel can reach once memory is taken away.
// Standalone; not part of libssm.so.
//   nvcc -gencode arch=compute_100a,code=sm_100a -O3 -o scan_core_rate scan_core_rate.cu && ./scan_core_rate
#include <cstdio>
#include <cuda_runtime.h>
__device__ __forceinline__ float ex2a(float v){float r;asm volatile("ex2.approx.ftz.f32 %0,%1;":"=f"(r):"f"(v));return r;}
__device__ __forceinline__ float lg2a(float v){float r;asm volatile("lg2.approx.ftz.f32 %0,%1;":"=f"(r):"f"(v));return r;}
__device__ __forceinline__ float rcpa(float v){float r;asm volatile("rcp.approx.ftz.f32 %0,%1;":"=f"(r):"f"(v));return r;}
template<bool PACKED, bool EPI>
__global__ void __launch_bounds__(64) core(float* out, const float* Ain, int steps, float seed){
  __shared__ float4 bc[32][8];
  const int lane=threadIdx.x&31;
  for(int i=threadIdx.x;i<32*8;i+=blockDim.x) ((float4*)bc)[i]=make_float4(0.01f*i,0.02f,0.03f,-0.01f*i);
  __syncthreads();
  float2 A[2][8], h[2][8];
  for(int c=0;c<2;c++) for(int k=0;k<8;k++){A[c][k]=make_float2(Ain[(c*8+k)*2+(threadIdx.x&1)], Ain[(c*8+k)*2+1]); h[c][k]=make_float2(0,0);}
  float dts0=seed+lane*1e-3f, dts1=seed*0.5f;
  float acc=0;
  for(int t=0;t<steps;t++){
    float dt0=dts0+t*1e-6f, dt1=dts1+t*1e-6f;
    if(EPI){ float e0=ex2a(-dt0), e1=ex2a(-dt1); dt0=lg2a(1.f+e0); dt1=lg2a(1.f+e1);} 
    const float4* row=bc[t&31];
    float2 dtc[2]={make_float2(dt0,dt0),make_float2(dt1,dt1)};
    float2 dtx[2]={make_float2(dt0*0.3f,dt0*0.3f),make_float2(dt1*0.7f,dt1*0.7f)};
    float2 ya[2]={make_float2(0,0),make_float2(0,0)}, yb[2]={make_float2(0,0),make_float2(0,0)};
#pragma unroll
    for(int q=0;q<4;q++){
      float4 bq=row[q], cq=row[4+q];
      float2 bp[2]={make_float2(bq.x,bq.y),make_float2(bq.z,bq.w)};
      float2 cp[2]={make_float2(cq.x,cq.y),make_float2(cq.z,cq.w)};
#pragma unroll
      for(int r=0;r<2;r++){ int k=2*q+r;
#pragma unroll
        for(int c=0;c<2;c++){
          if(PACKED){
            float2 v=__fmul2_rn(dtc[c],A[c][k]); float2 e=make_float2(ex2a(v.x),ex2a(v.y));
            h[c][k]=__ffma2_rn(e,h[c][k],__fmul2_rn(dtx[c],bp[r]));
            if(r==0) ya[c]=__ffma2_rn(cp[r],h[c][k],ya[c]); else yb[c]=__ffma2_rn(cp[r],h[c][k],yb[c]);
          } else {
            float vx=dtc[c].x*A[c][k].x, vy=dtc[c].y*A[c][k].y;
            float ex=ex2a(vx), ey=ex2a(vy);
            h[c][k].x=fmaf(ex,h[c][k].x,dtx[c].x*bp[r].x); h[c][k].y=fmaf(ey,h[c][k].y,dtx[c].y*bp[r].y);
            if(r==0){ya[c].x=fmaf(cp[r].x,h[c][k].x,ya[c].x); ya[c].y=fmaf(cp[r].y,h[c][k].y,ya[c].y);}
            else {yb[c].x=fmaf(cp[r].x,h[c][k].x,yb[c].x); yb[c].y=fmaf(cp[r].y,h[c][k].y,yb[c].y);}
          }
        }
      }
    }
    float y0=ya[0].x+ya[0].y+yb[0].x+yb[0].y, y1=ya[1].x+ya[1].y+yb[1].x+yb[1].y;
    if(EPI){ y0*=rcpa(1.f+ex2a(-y0)); y1*=rcpa(1.f+ex2a(-y1)); }
    acc+=y0+y1;
  }
  if(acc==1234.5f) out[threadIdx.x]=acc;
}
template<bool P,bool E> void run(const char* name, float* d, int sms, int steps){
  cudaEvent_t a,b; cudaEventCreate(&a); cudaEventCreate(&b);
  for(int bps: {2,4,5,6,8}){
    int grid=sms*bps;
    core<P,E><<<grid,64>>>(d,d+1024,steps,0.1f);
    cudaEventRecord(a); core<P,E><<<grid,64>>>(d,d+1024,steps,0.1f); cudaEventRecord(b); cudaEventSynchronize(b);
    float ms; cudaEventElapsedTime(&ms,a,b);
    double el=(double)grid*64*steps*32; // elements = threads*steps*2ch*16
    printf("%-26s CTAs/SM=%d warps/SM=%2d  %.3f ms  %.2f el/clk/SM @1965MHz\n",name,bps,2*bps,ms,el/(ms*1e-3)/(1.965e9*sms));
  }
}
int main(){ float* d; cudaMalloc(&d,8192); cudaMemset(d,0,8192); int sms=148; int steps=2000;
  run<true,false>("packed, core only",d,sms,steps);
  run<false,false>("scalar, core only",d,sms,steps);
  run<true,true>("packed, +softplus/silu",d,sms,steps);
  run<false,true>("scalar, +softplus/silu",d,sms,steps);
  cudaError_t e=cudaGetLastError(); printf("err=%s\n",cudaGetErrorString(e)); return e!=cudaSuccess; }
